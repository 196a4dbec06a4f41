"""The roofline arithmetic of bench.py against the layer's closed-form sizes:
one routed or shared expert of the dots3-note layer holds 3*H*F FP8 codes
plus its 128x128-block scales (23,598,720 bytes at H = 5120, F = 1536);
the gate/up GEMM reads the touched experts' gate and up weights, the
activation rows with their scales and writes h with its scales; the down
GEMM reads the down weights and h and writes y in bf16; FLOPs are
2 x rows x N x K of the real rows only. No GPU needed."""
import numpy as np

import bench
import gen


def _offsets(counts, shared):
    c = np.concatenate([np.asarray(counts, np.int64), [shared]])
    return np.concatenate([[0], np.cumsum(c)])


def test_decode_bytes_match_the_layer_sizes():
    wl = gen.WORKLOADS["decode"]
    sh = wl.shape
    T = 64
    per_gu = 2 * sh.F * sh.H + 2 * (sh.F // 128) * (sh.H // 128) * 4
    per_dn = sh.H * sh.F + (sh.H // 128) * (sh.F // 128) * 4
    assert per_gu + per_dn == 23_598_720               # one expert: codes + scales
    counts = np.zeros(sh.E, np.int64)
    counts[:207] = 2
    counts[207] = T * sh.K - 2 * 207                  # 208 touched routed experts
    w = bench.algorithmic_work(wl, T, _offsets(counts, T))
    rows = T * (sh.K + 1)
    assert w["touched_groups"] == 209                 # 208 routed + the shared expert
    assert w["bytes"]["gate_up"] == 209 * per_gu + rows * (sh.H + 4 * 40) + rows * (1536 + 4 * 12)
    assert w["bytes"]["down"] == 209 * per_dn + rows * (1536 + 4 * 12) + rows * sh.H * 2


def test_long_prefill_flops_count_real_rows_only():
    wl = gen.WORKLOADS["zipf"]
    sh = wl.shape
    T = 16384
    counts = np.full(sh.E, T * sh.K // sh.E, np.int64)
    w = bench.algorithmic_work(wl, T, _offsets(counts, T))
    rows = T * (sh.K + 1)
    assert w["flops"]["gate_up"] == 2.0 * rows * 3072 * 5120 == 4_638_564_679_680.0
    assert w["flops"]["down"] == 2.0 * rows * 5120 * 1536
    assert w["flops"]["gate_up"] + w["flops"]["down"] == 2.0 * T * 9 * 3 * 5120 * 1536   # 6.958 TFLOP


def test_fractions_divide_by_the_stated_peaks():
    work = {"bytes": {"route": 0, "permute": 0, "gate_up": 6_000_000_000, "down": 3_000_000_000, "combine": 0},
            "flops": {"gate_up": 3.0e12, "down": 1.5e12}}
    per = {"route": 0.0, "permute": 0.0, "gate_up": 1.0, "down": 0.5, "combine": 0.0}
    pk = {"hbm_gbs": 6000.0, "bf16_tflops": 1500.0, "bf16_tflops_sustained": 1500.0}
    f = bench.fractions(work, per, 1.5, pk)
    assert abs(f["gate_up"]["frac_hbm"] - 1.0) < 1e-9            # 6 GB in 1 ms = 6000 GB/s
    assert abs(f["gate_up"]["frac_fp8"] - 1.0) < 1e-9            # 3 TFLOP in 1 ms vs 2 x 1500
    assert f["binding"] in ("hbm", "tensor")
