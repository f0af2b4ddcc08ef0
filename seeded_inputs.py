"""Seeded synthetic inputs shared by the CUDA path's tests/benchmark and the oracle.

This module only draws numbers; it holds none of the method's arithmetic
(no quantisation, no layer math).  Every value is a pure function of
``(seed, stream, element index)``, so any slice of a tensor can be drawn on
its own: the oracle draws only the sequences it checks while the GPU side
draws the whole block, and both see identical values.

Generator: SplitMix64 (Steele, Lea and Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014) used as a counter-based mixer, followed by
the Box-Muller transform in float64 and a round-to-nearest-even conversion
to float16 (numpy's ``astype``).

Workload recipes follow the OPT-shaped configurations the pages describe
("FlexGen Guide: High-Throughput LLM Offloading on One GPU", section
"3. Group-Wise 4-Bit Quantization for Weights and KV Cache"; model family
from the OPT entry of the PIPO paper's reference list):
weights N(0, 0.02), biases 0, LayerNorm gamma 1 / beta 0, hidden states
N(0, 1); the quantize sweep adds 0.1 % outliers scaled x20 and some
constant groups.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_MASK = (1 << 64) - 1

# Stream identifiers: one independent stream per tensor role.
STREAM = {
    "wqkv": 1, "wo": 2, "w1": 3, "w2": 4,
    "bqkv": 5, "bo": 6, "b1": 7, "b2": 8,
    "ln1_g": 9, "ln1_b": 10, "ln2_g": 11, "ln2_b": 12,
    "prompt": 20, "decode": 21, "k_new": 22, "v_new": 23, "q": 24,
    "sweep": 30, "sweep_outlier": 31, "sweep_const": 32,
    "gemm_x": 40, "gemm_w": 41, "gemm_b": 42, "gemm_r": 43,
}


def _mix_scalar(z: int) -> int:
    z &= _MASK
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK
    return z ^ (z >> 31)


def stream_key(seed: int, stream: int) -> int:
    """64-bit key of one stream: two SplitMix64 finalisations of (seed, stream)."""
    return _mix_scalar(_mix_scalar(seed * 0x9E3779B97F4A7C15 + 1) ^ (stream * 0xD1B54A32D192ED03))


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def u64(key: int, start: int, count: int) -> np.ndarray:
    """Draws ``start .. start+count-1`` of the stream with the given key."""
    idx = np.arange(start, start + count, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(np.uint64(key) + (idx + np.uint64(1)) * _GOLDEN)


def _unit(z: np.ndarray) -> np.ndarray:
    # 53-bit uniform in (0, 1]
    return ((z >> np.uint64(11)).astype(np.float64) + 1.0) * (1.0 / 9007199254740992.0)


def normal64(key: int, start: int, count: int) -> np.ndarray:
    """Standard normals; element i uses draws 2i and 2i+1 of the stream."""
    z = u64(key, 2 * start, 2 * count)
    u1 = _unit(z[0::2])
    u2 = _unit(z[1::2])
    return np.sqrt(-2.0 * np.log(u1)) * np.cos(2.0 * np.pi * u2)


_POOL = None


def _pool() -> ThreadPoolExecutor:
    global _POOL
    if _POOL is None:
        _POOL = ThreadPoolExecutor(max_workers=max(1, min(16, os.cpu_count() or 1)))
    return _POOL


def normal_f16(seed: int, stream: int, shape, std: float = 1.0, start: int = 0) -> np.ndarray:
    """float16 array of N(0, std^2) draws; element i (row-major) is draw ``start + i``."""
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    key = stream_key(seed, stream)
    out = np.empty(n, dtype=np.float16)
    chunk = 1 << 22

    def work(lo: int) -> None:
        hi = min(n, lo + chunk)
        out[lo:hi] = (normal64(key, start + lo, hi - lo) * std).astype(np.float16)

    if n <= chunk:
        work(0)
    else:
        list(_pool().map(work, range(0, n, chunk)))
    return out.reshape(shape)


def constant_f16(shape, value: float) -> np.ndarray:
    return np.full(tuple(shape), value, dtype=np.float16)


# ----------------------------------------------------------------------------------------
# Workload recipes
# ----------------------------------------------------------------------------------------

def layer_weights_f16(seed: int, hidden: int, ffn: int, std: float = 0.02,
                      bias_std: float = 0.0, ln_random: bool = False) -> dict:
    """fp16 weights of one OPT decoder layer in ``[out, in]`` orientation.

    Default recipe: weights N(0, std^2), biases 0, LayerNorm gamma 1 and beta 0.
    ``bias_std`` > 0 and ``ln_random`` give non-trivial biases and LayerNorm
    parameters (used by the tests so that a dropped term shows up).
    """
    h, f = hidden, ffn
    w = {
        "wqkv": normal_f16(seed, STREAM["wqkv"], (3 * h, h), std),
        "wo": normal_f16(seed, STREAM["wo"], (h, h), std),
        "w1": normal_f16(seed, STREAM["w1"], (f, h), std),
        "w2": normal_f16(seed, STREAM["w2"], (h, f), std),
    }
    for name, n in (("bqkv", 3 * h), ("bo", h), ("b1", f), ("b2", h)):
        w[name] = (normal_f16(seed, STREAM[name], (n,), bias_std) if bias_std > 0
                   else np.zeros(n, dtype=np.float16))
    for name in ("ln1", "ln2"):
        if ln_random:
            w[name + "_g"] = (1.0 + normal_f16(seed, STREAM[name + "_g"], (h,), 0.1).astype(np.float32)).astype(np.float16)
            w[name + "_b"] = normal_f16(seed, STREAM[name + "_b"], (h,), 0.1)
        else:
            w[name + "_g"] = np.ones(h, dtype=np.float16)
            w[name + "_b"] = np.zeros(h, dtype=np.float16)
    return w


def hidden_rows(seed: int, stream: int, seq_ids, tokens_per_seq: int, hidden: int,
                token_start: int = 0, token_count: int | None = None) -> np.ndarray:
    """Hidden states ``[len(seq_ids), token_count, hidden]`` of N(0, 1).

    The full tensor of a stream is laid out as ``[seq, token, hidden]`` with
    ``tokens_per_seq`` tokens per sequence, so one sequence (or one token) can
    be drawn without drawing the others.
    """
    if token_count is None:
        token_count = tokens_per_seq - token_start
    out = np.empty((len(seq_ids), token_count, hidden), dtype=np.float16)
    for i, s in enumerate(seq_ids):
        start = (int(s) * tokens_per_seq + token_start) * hidden
        out[i] = normal_f16(seed, stream, (token_count, hidden), 1.0, start=start)
    return out


def hidden_block(seed: int, stream: int, num_seqs: int, tokens_per_seq: int, hidden: int) -> np.ndarray:
    """All sequences of :func:`hidden_rows` at once: ``[num_seqs, tokens_per_seq, hidden]``."""
    return normal_f16(seed, stream, (num_seqs, tokens_per_seq, hidden), 1.0)


def decode_inputs(seed: int, step: int, num_seqs: int, hidden: int, seq_ids=None) -> np.ndarray:
    """Fresh N(0, 1) hidden state per (decode step, sequence): ``[len(seq_ids), hidden]``."""
    if seq_ids is None:
        seq_ids = range(num_seqs)
    out = np.empty((len(seq_ids), hidden), dtype=np.float16)
    for i, s in enumerate(seq_ids):
        start = (int(step) * num_seqs + int(s)) * hidden
        out[i] = normal_f16(seed, STREAM["decode"], (hidden,), 1.0, start=start)
    return out


def sweep_tensor(seed: int, numel: int, row: int = 4096, group: int = 64) -> np.ndarray:
    """Quantize-sweep input ``[numel // row, row]``.

    N(0, 0.02); 0.1 % of elements (chosen by a seeded draw) scaled x20; 1 % of
    the groups overwritten by one constant; group 0 all zeros and group 1 a
    mix of +0 and -0.
    """
    assert numel % row == 0 and row % group == 0
    x = normal_f16(seed, STREAM["sweep"], (numel,), 0.02)
    okey = stream_key(seed, STREAM["sweep_outlier"])
    ckey = stream_key(seed, STREAM["sweep_const"])
    chunk = 1 << 22

    def work(lo: int) -> None:
        hi = min(numel, lo + chunk)
        sel = (u64(okey, lo, hi - lo) % np.uint64(1000)) == 0
        seg = x[lo:hi]
        seg[sel] = (seg[sel].astype(np.float32) * 20.0).astype(np.float16)
        g0, g1 = lo // group, hi // group
        gsel = (u64(ckey, g0, g1 - g0) % np.uint64(100)) == 0
        groups = seg.reshape(-1, group)
        groups[gsel] = groups[gsel][:, :1]

    if numel <= chunk:
        work(0)
    else:
        list(_pool().map(work, range(0, numel, chunk)))
    x[:group] = 0
    if numel >= 2 * group:
        x[group:2 * group] = np.where(np.arange(group) % 2 == 0, np.float16(0.0), np.float16(-0.0))
    return x.reshape(numel // row, row)
