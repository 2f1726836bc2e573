"""Seeded synthetic workloads for the fused chunked KL-distillation loss.

The source pages measure the loss on real student activations and a real
teacher cache (Llama 3.1 8B Instruct -> 3.2B student at 8K context, an
isolated output-projection benchmark at 32K/64K/256K, GPT-OSS 20B at 32 768
tokens).  None of those models or corpora exist here, so every workload is
drawn from the recipes below, with the pages' shapes:

* student hidden states ``H[T, d]`` ~ N(0, 1), rounded to bf16;
* output head ``W[V, d]`` ~ N(0, std) with std 0.02 (std d^-1/2 for the tiny
  case), rounded to bf16;
* the offline teacher cache per position: K distinct token ids drawn one at a
  time with Zipf(1.1) weights over the vocabulary, repeats rejected (that is,
  sampling without replacement, draw order kept), paired with log-probs made
  from K sorted-descending N(0, 2) draws passed through a log-softmax over K,
  so the k-th drawn id carries the k-th largest log-prob (the cache keeps the
  teacher's top-K most likely tokens per position, per "Дистилляция LLM на
  одной GPU: offline-кэш и chunked KL loss", section «Два приёма»);
* the GPT-OSS-shaped case draws half of each row's ids uniformly from the
  student's own top-200 logits ``W . h`` (computed in fp32 from the bf16
  inputs) and the other half from Zipf(1.1), excluding those;
* masks: trailing padding (5 % of the 8K row), or the last 1 % of each of
  eight packed 32 768-token sequences at 256K.

Random streams are drawn from one ``numpy.random.Generator(PCG64(seed))`` in
the fixed order H, W, teacher ids, teacher log-probs, mask, so both sides of
every parity test read identical arrays.  Nothing here computes the loss.
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "CONFIGS",
    "f32_to_bf16_bits",
    "bf16_bits_to_f32",
    "make_inputs",
    "make_config",
    "student_topk_numpy",
    "student_topk_torch",
]

# The five workloads, with the pages' shapes (T tokens, d hidden, V vocab,
# K cached teacher tokens per position, chunk rows per backward step).
CONFIGS = {
    "tiny": dict(T=256, d=64, V=1024, K=16, chunk=64, w_std=64 ** -0.5, mask=None),
    "8k": dict(T=8192, d=3072, V=128256, K=100, chunk=1024, w_std=0.02,
               mask=("tail", 410)),
    "32k": dict(T=32768, d=4096, V=128256, K=100, chunk=2048, w_std=0.02, mask=None),
    "oss": dict(T=32768, d=2880, V=201088, K=100, chunk=2048, w_std=0.02, mask=None,
                neighbourhood=(200, 50)),
    "256k": dict(T=262144, d=4096, V=128256, K=100, chunk=4096, w_std=0.02,
                 mask=("packed", 8, 32768, 328)),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (round to nearest, ties to even).

    Returns the 16-bit patterns as ``uint16``.  Inputs must be finite.
    """
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bit patterns to float32 (exact)."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32)
            << np.uint32(16)).view(np.float32)


def _normal_bf16(rng: np.random.Generator, rows: int, cols: int, std: float,
                 block_rows: int = 16384, fp32: bool = False) -> np.ndarray:
    out = np.empty((rows, cols), dtype=np.float32 if fp32 else np.uint16)
    s = np.float32(std)
    for r0 in range(0, rows, block_rows):
        r1 = min(rows, r0 + block_rows)
        x = rng.standard_normal((r1 - r0, cols), dtype=np.float32)
        if std != 1.0:
            x *= s
        out[r0:r1] = x if fp32 else f32_to_bf16_bits(x)
    return out


def _zipf_cdf(V: int, s: float) -> np.ndarray:
    w = np.arange(1, V + 1, dtype=np.float64) ** (-s)
    c = np.cumsum(w)
    return c / c[-1]


def _first_distinct(cand: np.ndarray, valid: np.ndarray, k: int):
    """Per row, the first ``k`` distinct valid candidates in draw order.

    Returns (out[n, k] int64 with -1 where a row ran short, count[n]).
    """
    n, m = cand.shape
    key = np.where(valid, cand, -1 - np.arange(m, dtype=np.int64)[None, :])
    order = np.argsort(key, axis=1, kind="stable")
    sk = np.take_along_axis(key, order, axis=1)
    first_sorted = np.ones(sk.shape, dtype=bool)
    first_sorted[:, 1:] = sk[:, 1:] != sk[:, :-1]
    first_sorted &= sk >= 0
    isfirst = np.zeros_like(first_sorted)
    np.put_along_axis(isfirst, order, first_sorted, axis=1)
    cnt = np.cumsum(isfirst, axis=1)
    take = isfirst & (cnt <= k)
    rows, cols = np.nonzero(take)
    out = np.full((n, k), -1, dtype=np.int64)
    out[rows, cnt[rows, cols] - 1] = cand[rows, cols]
    return out, np.minimum(cnt[:, -1], k)


def _zipf_distinct(rng: np.random.Generator, n: int, k: int, V: int, s: float,
                   exclude: np.ndarray | None = None, block_rows: int = 4096) -> np.ndarray:
    """Draw ``k`` distinct ids per row from Zipf(s) over [0, V), repeats rejected.

    ``exclude`` (n, e) lists ids a row may not take (they are rejected like
    repeats).  Candidates are drawn ``m`` at a time per row; a row that runs
    short draws further batches until it has ``k`` ids.
    """
    if k > V - (0 if exclude is None else exclude.shape[1]):
        raise ValueError("not enough distinct ids in the vocabulary")
    cdf = _zipf_cdf(V, s)
    out = np.empty((n, k), dtype=np.int32)
    m = 4 * k + 64
    for r0 in range(0, n, block_rows):
        r1 = min(n, r0 + block_rows)
        u = rng.random((r1 - r0, m))
        cand = np.minimum(np.searchsorted(cdf, u, side="right"), V - 1).astype(np.int64)
        ex = None if exclude is None else exclude[r0:r1]
        while True:
            valid = np.ones(cand.shape, dtype=bool)
            if ex is not None:
                valid = ~(cand[:, :, None] == ex[:, None, :]).any(axis=2)
            got, cnt = _first_distinct(cand, valid, k)
            short = np.nonzero(cnt < k)[0]
            if short.size == 0:
                break
            # Extend every row of the block by another batch (only short rows
            # use it; drawing for all keeps the stream layout simple).
            u = rng.random((r1 - r0, m))
            more = np.minimum(np.searchsorted(cdf, u, side="right"), V - 1).astype(np.int64)
            cand = np.concatenate([cand, more], axis=1)
        out[r0:r1] = got.astype(np.int32)
    return out


def student_topk_numpy(H_bits: np.ndarray, W_bits: np.ndarray, n: int,
                       block_rows: int = 256) -> np.ndarray:
    """Top-``n`` student logits ids per row, descending, from fp32 ``W . h``.

    Used only to build the GPT-OSS-shaped teacher cache at small sizes; the
    full-size case passes a GPU implementation of the same selection.
    """
    Wf = bf16_bits_to_f32(W_bits)
    T = H_bits.shape[0]
    out = np.empty((T, n), dtype=np.int64)
    for r0 in range(0, T, block_rows):
        r1 = min(T, r0 + block_rows)
        z = bf16_bits_to_f32(H_bits[r0:r1]) @ Wf.T
        part = np.argpartition(-z, n - 1, axis=1)[:, :n]
        zp = np.take_along_axis(z, part, axis=1)
        o = np.argsort(-zp, axis=1, kind="stable")
        out[r0:r1] = np.take_along_axis(part, o, axis=1)
    return out


def student_topk_torch(H_bits: np.ndarray, W_bits: np.ndarray, n: int,
                       block_rows: int = 1024) -> np.ndarray:
    """``student_topk_numpy`` on the GPU (torch, fp32 products, no TF32):
    the input recipe of the GPT-OSS-shaped teacher cache at full size."""
    import torch
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = False
    try:
        Wf = torch.from_numpy(W_bits.view(np.int16)).cuda().view(torch.bfloat16).float()
        out = np.empty((H_bits.shape[0], n), dtype=np.int64)
        for r0 in range(0, H_bits.shape[0], block_rows):
            r1 = min(H_bits.shape[0], r0 + block_rows)
            Hf = torch.from_numpy(H_bits[r0:r1].view(np.int16)).cuda().view(torch.bfloat16).float()
            z = Hf @ Wf.T
            out[r0:r1] = torch.topk(z, n, dim=1, sorted=True).indices.cpu().numpy()
            del z
        return out
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev


def _teacher_logp(rng: np.random.Generator, n: int, k: int, std: float) -> np.ndarray:
    vals = rng.standard_normal((n, k)) * std
    vals = -np.sort(-vals, axis=1)
    mx = vals[:, :1]
    lse = mx + np.log(np.exp(vals - mx).sum(axis=1, keepdims=True))
    return (vals - lse).astype(np.float32)


def _make_mask(rng: np.random.Generator, T: int, spec) -> np.ndarray | None:
    if spec is None:
        return None
    kind = spec[0]
    mask = np.ones(T, dtype=np.uint8)
    if kind == "tail":
        n = int(spec[1])
        if n > 0:
            mask[T - n:] = 0
    elif kind == "packed":
        nseq, seqlen, n = int(spec[1]), int(spec[2]), int(spec[3])
        if nseq * seqlen != T:
            raise ValueError("packed mask: nseq * seqlen != T")
        for s in range(nseq):
            mask[(s + 1) * seqlen - n:(s + 1) * seqlen] = 0
    elif kind == "bernoulli":
        frac = float(spec[1])
        mask = (rng.random(T) >= frac).astype(np.uint8)
    elif kind == "rows":
        mask[:] = 0
        mask[np.asarray(spec[1], dtype=np.int64)] = 1
    elif kind == "none":
        mask[:] = 0
    elif kind == "ones":
        pass
    else:
        raise ValueError(f"unknown mask spec {spec!r}")
    return mask


def make_inputs(T: int, d: int, V: int, K: int, *, seed: int = 0, h_std: float = 1.0,
                w_std: float = 0.02, teacher_std: float = 2.0, zipf_s: float = 1.1,
                mask=None, neighbourhood=None, student_topk=None, chunk: int | None = None,
                name: str = "custom", fp32: bool = False) -> dict:
    """Draw one workload.

    Returns a dict with ``H`` (uint16 bf16 bits, [T, d]), ``W`` (uint16 bf16
    bits, [V, d]), ``idx`` (int32 [T, K]), ``logp`` (float32 [T, K]), ``mask``
    (uint8 [T] or None = every position counts) and the sizes.  ``fp32``:
    H and W are the same draws kept in float32, not rounded to bf16.
    ``neighbourhood=(top, take)`` draws ``take`` ids per row uniformly from the
    row's top-``top`` student logits (``student_topk(H, W, top)`` returns them,
    descending) and the remaining ``K - take`` from Zipf, excluding those.
    """
    if fp32 and neighbourhood is not None:
        raise ValueError("the student top-n neighbourhood is drawn from bf16 inputs")
    rng = np.random.Generator(np.random.PCG64(seed))
    H = _normal_bf16(rng, T, d, h_std, fp32=fp32)
    W = _normal_bf16(rng, V, d, w_std, fp32=fp32)
    if neighbourhood is None:
        idx = _zipf_distinct(rng, T, K, V, zipf_s) if T > 0 else np.empty((0, K), np.int32)
    else:
        top, take = neighbourhood
        if take > K or top > V:
            raise ValueError("bad neighbourhood spec")
        fn = student_topk if student_topk is not None else student_topk_numpy
        nb = np.asarray(fn(H, W, top), dtype=np.int64)           # [T, top], descending z
        keys = rng.random((T, top))
        pick = np.sort(np.argsort(keys, axis=1, kind="stable")[:, :take], axis=1)
        chosen = np.take_along_axis(nb, pick, axis=1)            # descending z order
        rest = _zipf_distinct(rng, T, K - take, V, zipf_s, exclude=chosen)
        idx = np.concatenate([chosen.astype(np.int32), rest], axis=1)
    logp = _teacher_logp(rng, T, K, teacher_std)
    m = _make_mask(rng, T, mask)
    return dict(name=name, seed=seed, T=T, d=d, V=V, K=K,
                chunk=chunk if chunk is not None else max(1, T),
                H=H, W=W, idx=np.ascontiguousarray(idx, dtype=np.int32),
                logp=np.ascontiguousarray(logp, dtype=np.float32), mask=m)


def make_config(name: str, seed: int = 0, student_topk=None, fp32: bool = False) -> dict:
    """One of the five named workloads (see ``CONFIGS``); ``fp32`` keeps H
    and W in float32 (the tiny workload is an fp32 case)."""
    c = dict(CONFIGS[name])
    return make_inputs(c["T"], c["d"], c["V"], c["K"], seed=seed, w_std=c["w_std"],
                       mask=c.get("mask"), neighbourhood=c.get("neighbourhood"),
                       student_topk=student_topk, chunk=c["chunk"], name=name, fp32=fp32)
