"""Host arithmetic of bench.py (CPU): the algorithmic bytes each kernel's
roofline divides by, and the roofline objects built from them, against the
per-element figures the kernels are defined by (a 16-element NVFP4 block is
16 input elements, 8 packed bytes and one scale byte)."""
import types

import pytest
import torch

import bench
import workloads


def test_algorithmic_bytes_per_element():
    w = workloads.WEIGHT_4K  # bf16, 4096 x 4096
    n = w.numel
    ab = bench.algorithmic_bytes(w)
    per = {k: v / n for k, v in ab.items()}
    assert per["amax"] == 2.0                           # read x
    assert per["nvfp4_quantize"] == 2 + 1 / 2 + 1 / 16  # read x, write codes and E4M3 scales
    assert per["mxfp4_quantize"] == 2 + 1 / 2 + 1 / 32  # read x, write codes and E8M0 scales
    assert per["nvfp4_dequantize"] == 1 / 2 + 1 / 16 + 2
    assert per["mxfp4_dequantize"] == 1 / 2 + 1 / 32 + 2
    assert per["scale_search"] == per["nvfp4_quantize"]
    assert per["scales_to_mma"] == 2 / 16               # read and write one byte per block
    f32 = workloads.TINY_F32
    assert bench.algorithmic_bytes(f32)["amax"] == 4 * f32.numel


def test_gemm_roofline_uses_the_fp4_peak():
    pk = {"hbm_gbs": 6538.0, "sm_max_mhz": 1965.0, "bf16_tflops": 1642.8, "source": "measured"}
    M, N, K = 8192, 4096, 14336
    r = bench.roofline_for("nvfp4_gemm", {"us": 312.0}, workloads.GEMM_ACT, pk, gemm_mnk=(M, N, K))
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["peak"] == pytest.approx(4 * 1642.8, abs=0.05)
    assert r["achieved"] == pytest.approx(2 * M * N * K / 312e-6 / 1e12, abs=0.05)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"], abs=1e-4)


def test_hbm_roofline_is_the_kernel_bandwidth_over_the_copy_peak():
    pk = {"hbm_gbs": 6538.0, "sm_max_mhz": 1965.0, "bf16_tflops": 1642.8, "source": "measured"}
    k = {"us": 41.1, "gbs": 5712.0, "frac_hbm": round(5712.0 / 6538.0, 4)}
    r = bench.roofline_for("amax", k, workloads.ACT_8K, pk)
    assert (r["bound"], r["unit"], r["achieved"], r["peak"]) == ("hbm", "GB/s", 5712.0, 6538.0)
    assert r["frac"] == k["frac_hbm"]


def test_search_roofline_counts_fp32_lane_operations(monkeypatch):
    """The ALU bound: distinct candidate evaluations x 16 elements x the
    fp32 operations of one evaluation, against SMs x 128 lanes x clock."""
    pk = {"hbm_gbs": 6538.0, "sm_max_mhz": 1965.0, "bf16_tflops": 1642.8, "source": "measured"}
    monkeypatch.setattr(torch.cuda, "current_device", lambda: 0)
    monkeypatch.setattr(torch.cuda, "get_device_properties",
                        lambda i: types.SimpleNamespace(multi_processor_count=148))
    n_cand = 5_407_393
    r = bench.roofline_for("scale_search", {"us": 35.3}, workloads.WEIGHT_4K, pk, n_cand=n_cand)
    assert r["bound"] == "alu"
    assert r["peak"] == pytest.approx(148 * 128 * 1965e6 / 1e12, abs=0.01)
    assert r["achieved"] == pytest.approx(n_cand * 16 * bench.SEARCH_OPS_PER_EVAL / 35.3e-6 / 1e12, abs=1e-3)


def test_search_candidate_count_matches_its_definition():
    """The candidates of a block are the contiguous E4M3 codes from the one
    nearest 0.7 A_b/(6g) to the one nearest A_b/(6g): counted here block by
    block with the E4M3 rounding written out (nearest value, ties to the
    even code), against the vectorised count the bench uses."""
    g_ = torch.Generator().manual_seed(3)
    x = (torch.randn(64, 256, generator=g_) * 0.05).to(torch.bfloat16)
    amax = x.float().abs().max().item()
    g = float(torch.tensor(amax / 2688.0, dtype=torch.float32))
    vals = torch.arange(127, dtype=torch.uint8).view(torch.float8_e4m3fn).double()

    def nearest(t: float) -> int:
        t = min(t, 448.0)
        d = (vals - t).abs()
        best = int(d.argmin())
        ties = (d == d[best]).nonzero().flatten().tolist()
        return min(ties, key=lambda c: (c & 1, c)) if len(ties) > 1 else best

    ab = x.float().abs().reshape(-1, 16).amax(dim=1).double()
    want = 0
    for a in ab.tolist():
        t_hi = float(torch.tensor(a / (6.0 * g), dtype=torch.float32))
        t_lo = float(torch.tensor(a * 147.0 / (1260.0 * g), dtype=torch.float32))
        want += nearest(t_hi) - nearest(t_lo) + 1
    assert bench.search_candidate_count(x, g) == want


def test_layer_spans_cover_the_weight_set_once():
    sizes = [r * c for r, c in workloads.MODEL_MATRICES] * workloads.MODEL_LAYERS
    per = len(workloads.MODEL_MATRICES)
    spans = bench.layer_spans(sizes, per)
    assert len(spans) == workloads.MODEL_LAYERS
    assert spans[0][0] == 0 and spans[0][2] == 0 and spans[-1][3] == workloads.model_numel()
    for (li, n, e0, e1), nxt in zip(spans, spans[1:] + [None]):
        assert n == per and e1 - e0 == sum(sizes[li:li + n])
        if nxt is not None:
            assert nxt[0] == li + n and nxt[2] == e1  # contiguous, no gap, no overlap
    # a short last group
    assert bench.layer_spans([3, 4, 5, 6, 7], 2) == [(0, 2, 0, 7), (2, 2, 7, 18), (4, 1, 18, 25)]
