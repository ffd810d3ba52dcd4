"""Seeded synthetic verification workloads (shared by tests, bench and smoke).

This module only *draws inputs*: logits, drafted ids, draft lengths and the
uniforms the verification rule consumes.  It contains none of the rule's own
arithmetic.  Drafted ids are sampled the way a drafter would produce them
(Gumbel-max over the stored draft logits, or the n-gram recipe for the
one-hot configuration); that is drafter behaviour, outside the verified path.

The five named workloads stand in for the pages' RL rollout workloads (their
datasets and models are not available here):

1 tiny sanity          B=4,   k=4,  V=1000,    fp32, T=1,   Z~N(0,2^2), Y=Z+N(0,0.3^2)
2 quantized self-draft B=64,  k=8,  V=151936,  bf16, T=1,   Z~N(0,1)+8 on a favoured id, Y=Z+N(0,0.2^2)
3 n-gram / one-hot     B=128, k=16, V=151936,  bf16, T=1,   Z~N(0,1)+6; no draft logits; x = favoured id w.p. 0.8 else uniform
4 long-tail straggler  B=8,   k=24, V=151936,  bf16, T=0.6, Z~N(0,1.5^2)+10, Y=Z+N(0,0.15^2)
5 length-aware budgets B=256, k_max=12, V=128256, fp32, T=1, L in {0,4,12} w.p. .5/.3/.2,
                       Z~N(0,1)+7, Y=Z+N(0,0.25^2), padded rows filled with NaN

Seeds: 92*1000 + config; numpy ``SeedSequence(seed).spawn(6)`` gives the
sub-streams 0 target logits, 1 draft noise, 2 favoured ids, 3 draft-token draws,
4 uniforms, 5 draft lengths.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

F32 = "f32"
BF16 = "bf16"


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 (round to nearest even); returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    rounding = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    out = ((u + rounding) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclass
class Workload:
    name: str
    B: int
    k_max: int
    V: int
    dtype: str                 # "f32" | "bf16"
    temperature: float
    target: np.ndarray         # float32 or uint16 (bf16 bits) [B, k_max+1, row_stride]
    draft: np.ndarray | None   # same dtype [B, k_max, row_stride] or None (one-hot q)
    tokens: np.ndarray         # int32 [B, k_max]; -1 beyond each request's length
    lens: np.ndarray | None    # int32 [B] or None (every request uses k_max)
    uniforms: np.ndarray       # float32 [B, k_max+1] in [0, 1)
    favoured: np.ndarray = field(repr=False, default=None)  # int32 [B, k_max+1]
    row_stride: int = 0

    @property
    def draft_lens(self) -> np.ndarray:
        if self.lens is None:
            return np.full(self.B, self.k_max, np.int32)
        return self.lens

    @property
    def positions(self) -> int:
        """Draft positions submitted for verification in one call."""
        return int(self.draft_lens.sum())

    @property
    def esize(self) -> int:
        return 4 if self.dtype == F32 else 2


def _store(values_f32: np.ndarray, dtype: str) -> np.ndarray:
    return values_f32.astype(np.float32) if dtype == F32 else f32_to_bf16_bits(values_f32)


def _as_f32(stored: np.ndarray, dtype: str) -> np.ndarray:
    return stored.astype(np.float32) if dtype == F32 else bf16_bits_to_f32(stored)


def make_workload(*, B: int, k_max: int, V: int, dtype: str = F32,
                  temperature: float = 1.0, seed: int = 0,
                  z_sigma: float = 1.0, boost: float = 0.0,
                  draft_mode: str = "logits",        # "logits" | "ids"
                  draft_noise: float = 0.2, fav_prob: float = 0.8,
                  lens_choices=None, lens_probs=None, lens=None,
                  pad_value: float = float("nan"), row_stride: int | None = None,
                  name: str = "custom") -> Workload:
    """Draw one seeded workload.  Only rows a request uses are drawn; padded
    rows (beyond ``lens[b]``) and the padding columns of a wider
    ``row_stride`` hold ``pad_value`` (NaN by default) and must never be read."""
    if row_stride is None:
        row_stride = V
    assert row_stride >= V
    ss = np.random.SeedSequence(seed)
    rng_t, rng_noise, rng_fav, rng_x, rng_u, rng_len = [np.random.Generator(np.random.PCG64(s)) for s in ss.spawn(6)]

    if lens is not None:
        lens_arr = np.asarray(lens, np.int32).reshape(B)
    elif lens_choices is not None:
        lens_arr = rng_len.choice(np.asarray(lens_choices, np.int32), size=B, p=lens_probs).astype(np.int32)
    else:
        lens_arr = None
    L_of = (lambda b: k_max) if lens_arr is None else (lambda b: int(lens_arr[b]))

    favoured = rng_fav.integers(0, V, size=(B, k_max + 1), dtype=np.int64).astype(np.int32)
    store_dt = np.float32 if dtype == F32 else np.uint16
    pad_stored = _store(np.array([pad_value], np.float32), dtype)[0]
    target = np.full((B, k_max + 1, row_stride), pad_stored, dtype=store_dt)
    draft = None
    if draft_mode == "logits" and k_max > 0:
        draft = np.full((B, k_max, row_stride), pad_stored, dtype=store_dt)
    tokens = np.full((B, k_max), -1, np.int32)

    for b in range(B):
        L = L_of(b)
        z = rng_t.standard_normal((L + 1, V), dtype=np.float32)
        z *= np.float32(z_sigma)
        if boost:
            z[np.arange(L + 1), favoured[b, :L + 1]] += np.float32(boost)
        target[b, :L + 1, :V] = _store(z, dtype)
        if L == 0:
            continue
        if draft_mode == "logits":
            y = z[:L] + rng_noise.standard_normal((L, V), dtype=np.float32) * np.float32(draft_noise)
            y_stored = _store(y, dtype)
            draft[b, :L, :V] = y_stored
            # Drafter: sample x_i from softmax(Y_i / T) of the stored draft
            # logits with the Gumbel-max trick.
            g = rng_x.random((L, V), dtype=np.float64)
            with np.errstate(divide="ignore"):
                gumbel = -np.log(-np.log(g))
            scores = _as_f32(y_stored, dtype).astype(np.float64) / temperature + gumbel
            tokens[b, :L] = np.argmax(scores, axis=1).astype(np.int32)
        else:
            # n-gram / suffix drafter: the favoured id w.p. fav_prob, else a
            # uniformly random id.
            pick = rng_x.random(L) < fav_prob
            rand_ids = rng_x.integers(0, V, size=L, dtype=np.int64).astype(np.int32)
            tokens[b, :L] = np.where(pick, favoured[b, :L], rand_ids)

    uniforms = rng_u.random((B, k_max + 1), dtype=np.float32)
    return Workload(name=name, B=B, k_max=k_max, V=V, dtype=dtype,
                    temperature=float(temperature), target=target, draft=draft,
                    tokens=tokens, lens=lens_arr, uniforms=uniforms,
                    favoured=favoured, row_stride=row_stride)


CONFIGS = {
    1: dict(name="tiny-sanity", B=4, k_max=4, V=1000, dtype=F32, temperature=1.0,
            z_sigma=2.0, boost=0.0, draft_mode="logits", draft_noise=0.3),
    2: dict(name="quantized-self-draft", B=64, k_max=8, V=151936, dtype=BF16,
            temperature=1.0, z_sigma=1.0, boost=8.0, draft_mode="logits", draft_noise=0.2),
    3: dict(name="ngram-one-hot", B=128, k_max=16, V=151936, dtype=BF16,
            temperature=1.0, z_sigma=1.0, boost=6.0, draft_mode="ids", fav_prob=0.8),
    4: dict(name="long-tail-straggler", B=8, k_max=24, V=151936, dtype=BF16,
            temperature=0.6, z_sigma=1.5, boost=10.0, draft_mode="logits", draft_noise=0.15),
    5: dict(name="length-aware-budgets", B=256, k_max=12, V=128256, dtype=F32,
            temperature=1.0, z_sigma=1.0, boost=7.0, draft_mode="logits", draft_noise=0.25,
            lens_choices=(0, 4, 12), lens_probs=(0.5, 0.3, 0.2)),
}


def config_seed(cfg: int) -> int:
    return 92 * 1000 + cfg


def make_config(cfg: int, **overrides) -> Workload:
    """One of the five named workloads, drawn from its fixed seed."""
    params = dict(CONFIGS[cfg])
    params.update(overrides)
    return make_workload(seed=config_seed(cfg), **params)
