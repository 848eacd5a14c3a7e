"""Seeded synthetic inputs for the fused chunked KL loss.

This module is shared by the CUDA path's tests/benchmark and by the CPU oracle.
It draws random numbers and rounds them to the storage types; it holds none of
the loss arithmetic.

Workload shapes follow the pages' workloads:
  * "Llama 3.1 8B teacher -> ~3.2B student, 8K context" (AI Trends summary of
    the paper, figure descriptions and evidence list),
  * "32K tokens, toy output projection" and "256K tokens" (aibase.it write-up
    "Knowledge Distillation 비용 줄이기", section "chunked KL loss가 하는 일"),
  * "gpt-oss vocabulary 201,088, sequence 32K, batch 4" (same write-up,
    section "문제가 되는 지점"),
with the top-100 teacher cache of section "offline top-K logits 방식".

Recipe (all streams are children of ``np.random.SeedSequence(1000 + cfg)``):
  stream 0  hidden   f32 standard normal, row-major [N, H], rounded to bf16 (RNE)
  stream 1  W        f32 normal(0, 0.02), [V, H], rounded to bf16 (RNE)
  stream 2  ids      per row K distinct ids, uniform in [0, V): a row of K
                     uniform integers is redrawn whole until it has no repeat
                     (exact rejection sampling of an ordered distinct K-tuple);
                     when K^2 > 2V each row is drawn without replacement instead
  stream 3  logits   f32 normal(0, sigma), [N, K], each row sorted descending
                     and paired with the ids in draw order
  stream 4  mask     exactly round(f * N) rows set to 0, chosen without
                     replacement; the rest are 1
  stream 5  sample   the sampled valid rows used for per-row checks
Large arrays are drawn in fixed blocks of rows so that memory stays bounded;
the block size is part of the recipe.
"""
from __future__ import annotations

import dataclasses
import numpy as np

__all__ = ["Config", "CONFIGS", "Inputs", "make_inputs", "make_custom", "make_sampled_targets",
           "f32_to_bf16_bits", "bf16_bits_to_f32", "sample_rows"]

_BLOCK_ELEMS = 1 << 24


@dataclasses.dataclass(frozen=True)
class Config:
    name: str
    N: int
    H: int
    V: int
    K: int
    T: float
    chunk: int          # 0 = library's automatic choice
    sigma: float        # std-dev of the teacher logits
    mask_frac: float
    seed: int

    @property
    def n_masked(self) -> int:
        return int(round(self.mask_frac * self.N))


CONFIGS = {
    0: Config("tiny_N256_H256_V4096_K16", 256, 256, 4096, 16, 1.0, 64, 2.0, 0.0, 1000),
    1: Config("llama8b_to_3b_8k_N8192_H3072_V128256_K100", 8192, 3072, 128256, 100, 1.0, 0, 3.0, 0.05, 1001),
    2: Config("toyproj_32k_N32768_H4096_V128256_K100", 32768, 4096, 128256, 100, 1.0, 1024, 3.0, 0.0, 1002),
    3: Config("gptoss20b_4x32k_N131072_H2880_V201088_K100", 131072, 2880, 201088, 100, 1.0, 0, 3.0, 0.03, 1003),
    4: Config("scale_256k_N262144_H4096_V128256_K100_T2", 262144, 4096, 128256, 100, 2.0, 2048, 3.0, 0.10, 1004),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bfloat16 with round-to-nearest-even; returns uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    b = x.view(np.uint32)
    rounding = np.uint32(0x7FFF) + ((b >> np.uint32(16)) & np.uint32(1))
    out = ((b + rounding) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        out[nan] = np.uint16(0x7FC0)
    return out


def bf16_bits_to_f32(u: np.ndarray) -> np.ndarray:
    """Exact widening of bfloat16 bits to float32."""
    u = np.ascontiguousarray(u, dtype=np.uint16)
    return (u.astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Inputs:
    cfg: Config
    hidden: np.ndarray      # uint16 bf16 bits [N, H]
    W: np.ndarray           # uint16 bf16 bits [V, H]
    topk_idx: np.ndarray    # int32 [N, K]
    topk_logit: np.ndarray  # float32 [N, K]
    row_mask: np.ndarray    # uint8 [N]


def _normal_bf16(rng: np.random.Generator, rows: int, cols: int, scale: float) -> np.ndarray:
    out = np.empty((rows, cols), dtype=np.uint16)
    step = max(1, _BLOCK_ELEMS // max(cols, 1))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        x = rng.standard_normal((r1 - r0, cols), dtype=np.float32)
        if scale != 1.0:
            x *= np.float32(scale)
        out[r0:r1] = f32_to_bf16_bits(x)
    return out


def _distinct_ids(rng: np.random.Generator, rows: int, V: int, K: int) -> np.ndarray:
    if K * K > 2 * V:  # repeats would be common: draw each row without replacement
        return np.stack([rng.choice(V, size=K, replace=False) for _ in range(rows)]).astype(np.int32)
    ids = rng.integers(0, V, size=(rows, K), dtype=np.int64)
    while True:
        s = np.sort(ids, axis=1)
        bad = np.nonzero((s[:, 1:] == s[:, :-1]).any(axis=1))[0] if K > 1 else np.zeros(0, np.int64)
        if bad.size == 0:
            break
        ids[bad] = rng.integers(0, V, size=(bad.size, K), dtype=np.int64)
    return ids.astype(np.int32)


def make_custom(N: int, H: int, V: int, K: int, T: float = 1.0, sigma: float = 3.0,
                mask_frac: float = 0.0, seed: int = 0, chunk: int = 0,
                name: str = "custom") -> Inputs:
    cfg = Config(name, N, H, V, K, T, chunk, sigma, mask_frac, seed)
    return make_inputs(cfg)


def make_inputs(cfg: Config | int) -> Inputs:
    if isinstance(cfg, int):
        cfg = CONFIGS[cfg]
    ss = np.random.SeedSequence(cfg.seed)
    r_h, r_w, r_id, r_lg, r_m, _ = [np.random.Generator(np.random.PCG64(s)) for s in ss.spawn(6)]
    hidden = _normal_bf16(r_h, cfg.N, cfg.H, 1.0)
    W = _normal_bf16(r_w, cfg.V, cfg.H, 0.02)
    ids = np.empty((cfg.N, cfg.K), dtype=np.int32)
    logit = np.empty((cfg.N, cfg.K), dtype=np.float32)
    step = max(1, _BLOCK_ELEMS // max(cfg.K, 1))
    for r0 in range(0, cfg.N, step):
        r1 = min(cfg.N, r0 + step)
        ids[r0:r1] = _distinct_ids(r_id, r1 - r0, cfg.V, cfg.K)
    for r0 in range(0, cfg.N, step):
        r1 = min(cfg.N, r0 + step)
        x = r_lg.standard_normal((r1 - r0, cfg.K), dtype=np.float32) * np.float32(cfg.sigma)
        logit[r0:r1] = -np.sort(-x, axis=1)
    mask = np.ones(cfg.N, dtype=np.uint8)
    m = cfg.n_masked
    if m > 0:
        mask[r_m.choice(cfg.N, size=m, replace=False)] = 0
    return Inputs(cfg, hidden, W, ids, logit, mask)


def sample_rows(inp: Inputs, n: int = 64) -> np.ndarray:
    """Seeded choice of ``n`` valid (unmasked) rows, sorted ascending."""
    ss = np.random.SeedSequence(inp.cfg.seed)
    r_s = np.random.Generator(np.random.PCG64(ss.spawn(6)[5]))
    valid = np.nonzero(inp.row_mask)[0]
    n = min(n, valid.size)
    return np.sort(r_s.choice(valid, size=n, replace=False)).astype(np.int64)


def make_sampled_targets(N: int, H: int, V: int, K: int, T: float = 1.0, sigma: float = 3.0,
                         mask_frac: float = 0.0, seed: int = 0, chunk: int = 0) -> Inputs:
    """Sparse sampled teacher targets (RS-KD form): per row a synthetic teacher
    over a candidate set of min(4K, V) distinct ids with logits N(0, sigma),
    K ids drawn WITH replacement from it, and one positive weight per draw
    (uniform in [0.5, 1.5)); ``topk_logit`` holds those weights.  hidden, W and
    the mask follow the usual recipe (streams 0, 1, 4); stream 2 draws the
    candidates and samples, stream 3 the candidate logits and the weights."""
    base = make_custom(N, H, V, 1, T=T, sigma=sigma, mask_frac=mask_frac, seed=seed, chunk=chunk,
                       name="sampled_targets")
    ss = np.random.SeedSequence(seed)
    _, _, r_id, r_lg, _, _ = [np.random.Generator(np.random.PCG64(x)) for x in ss.spawn(6)]
    C = min(4 * K, V)
    ids = np.empty((N, K), np.int32)
    w = np.empty((N, K), np.float32)
    for r in range(N):
        cand = r_id.choice(V, size=C, replace=False)
        lg = r_lg.standard_normal(C) * sigma
        pr = np.exp(lg - lg.max())
        pr /= pr.sum()
        ids[r] = cand[r_id.choice(C, size=K, replace=True, p=pr)]
        w[r] = r_lg.uniform(0.5, 1.5, K).astype(np.float32)
    cfg = dataclasses.replace(base.cfg, K=K)
    return Inputs(cfg, base.hidden, base.W, ids, w, base.row_mask)
