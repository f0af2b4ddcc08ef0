"""The benchmark's algorithmic work per kernel (the numerators of every roofline fraction)
against per-unit figures stated independently of it: OPT layer FLOPs (24 S h^2 for the four
GEMMs with F = 4h), 4-bit bytes (0.5625 per weight: half a byte of code plus 4 bytes of fp16
min and scale per 64), 144 bytes of K and V per cached token at head_dim 128."""
import importlib.util
import os

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def test_opt6p7b_decode_step_work(bench):
    wl = bench.WORKLOADS["opt-6.7b-layer"]
    S, h, H = 512, 4096, 32
    work, totals = bench.kernel_work(wl, S, 512)
    gemm = sum(w for b, w in work.values() if b == "tensor")
    assert gemm == 24 * S * h * h                        # 206 GFLOP per step
    assert totals["kv_bytes_per_token"] == 2 * (64 + 4 * 2) == 144
    assert totals["w4_bytes"] == 12 * h * h * 9 // 16   # 113.2 MB
    att = work["attention"][1]
    # 1.208 GB of KV4 read, q in and o out, and the fused append: k, v in, their codes out
    assert att == S * H * 512 * 144 + 2 * S * h * 2 + 2 * S * h * 2 + S * H * 144
    assert work["kv_append"][1] == S * 2 * h * 2 + S * 2 * (h // 2 + h // 16)
    # a block this large appends in its own kernel: the attention reads the cache, q and o only
    work, _ = bench.kernel_work(wl, S, 512, fused_append=False)
    assert work["attention"][1] == S * H * 512 * 144 + 2 * S * h * 2
    units = bench.kernel_units(wl, S, 512)
    assert units["attention"] == S * H * 512            # traffic of a smaller capture scales by these


def test_stack_and_prefill_shapes(bench):
    for name, layers in (("opt-30b-stack", 48), ("opt-175b-stack", 16)):
        wl = bench.WORKLOADS[name]
        assert wl["hidden"] % wl["heads"] == 0 and wl["ffn"] == 4 * wl["hidden"]
        assert wl["layers"] == layers
    wl = bench.WORKLOADS["opt-175b-stack"]
    assert wl["nb"] * wl["gbs"] == 256 and wl["model_layers"] == 96
    # prefill: row t of a prompt reads t + 1 cached tokens, so P rows read P (P + 1) / 2 in all
    wl = bench.WORKLOADS["opt-6.7b-prefill"]
    P = wl["prompt"]
    work, _ = bench.kernel_work(wl, P, (P + 1) / 2, fused_append=False)
    assert work["attention"][1] == pytest.approx(wl["heads"] * P * (P + 1) / 2 * 144 + 2 * P * wl["hidden"] * 2)


def test_w4a8_decode_step_work(bench):
    # the W4A8 form: the same 24 S h^2 of products, now integer ("tensor_i8", against the int8
    # peak), and the activation quantisers of the attention and ReLU outputs: fp16 in, int8 and
    # one fp32 scale per row out
    wl = bench.WORKLOADS["opt-6.7b-layer-w4a8"]
    S, h, F = 512, 4096, 16384
    work, _ = bench.kernel_work(wl, S, 512)
    assert sum(w for b, w in work.values() if b == "tensor_i8") == 24 * S * h * h
    assert not any(b == "tensor" for b, _ in work.values())
    assert work["out_act8"] == ("hbm", S * h * 3 + S * 4)
    assert work["fc2_act8"] == ("hbm", S * F * 3 + S * 4)
    assert bench.kernel_units(wl, S, 512)["fc2_act8"] == S
