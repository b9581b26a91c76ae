"""bench.py's host-side arithmetic (no GPU): the algorithmic FLOPs and bytes that every roofline
fraction divides by, checked against the per-token counts that follow from the layer's shapes
("Gate projection" page: three 7168 x 2048 projections per expert; eight routed experts and one
shared per token at the DeepSeek-V3.2 shape; the router's 7168 x 256 product)."""
import numpy as np

import bench
import synthetic


def test_flops_per_token_of_the_workloads():
    # 3 projections x 2 FLOP x d x inter per SwiGLU, k routed + the shared ones, plus the router
    assert synthetic.CONFIGS["C3"].flops_per_token() == 2 * 7168 * 2048 * 3 * 9 + 2 * 7168 * 256 == 796_393_472
    assert synthetic.CONFIGS["C4"].flops_per_token() == 796_393_472
    assert synthetic.CONFIGS["C2"].flops_per_token() == 2 * 2048 * 1024 * 3 * (6 + 2) + 2 * 2048 * 64 == 100_925_440
    assert synthetic.CONFIGS["C1"].flops_per_token() == 2 * 256 * 128 * 3 * (2 + 1) + 2 * 256 * 8 == 593_920
    # the dense block: the MLP alone, no router
    assert synthetic.CONFIGS["D1"].flops_per_token() == 2 * 7168 * 18432 * 3


def test_work_of_the_prefill_step_and_its_up_gemm():
    s = synthetic.CONFIGS["C4"]
    w = bench.work(s, np.full(256, 512))      # every expert touched
    T, d, I = 16384, 7168, 2048
    assert w["touched"] == 256
    assert w["step_flops"] == T * 796_393_472
    assert w["up_flops"] == 2 * d * 2 * I * T * 8 + 2 * d * 2 * I * T          # w1|w3 of 8 routed + the shared
    scales = lambda r, c: (r // 128) * (c // 128) * 4
    expert = 3 * d * I + 2 * scales(I, d) + scales(d, I)                           # FP8 bytes + fp32 block scales
    assert w["step_bytes"] == 256 * expert + expert + 256 * d * 2 + 4 * T * d * 2
    # bf16 activations double the activation bytes of the up GEMM, not its weight bytes
    w16 = bench.work(s, np.full(256, 512), act8=False)
    act8 = (T * 8 + T) * d + (T * 8 * I + T * I)
    assert w16["up_bytes"] - w["up_bytes"] == act8


def test_decode_counts_only_touched_experts():
    s = synthetic.CONFIGS["C3"]
    counts = np.zeros(256, int)
    counts[:200] = 5
    w = bench.work(s, counts)
    full = bench.work(s, np.full(256, 4))
    assert w["touched"] == 200
    per_expert = (full["step_bytes"] - w["step_bytes"]) / 56
    assert per_expert == 3 * 7168 * 2048 + 3 * 16 * 56 * 4
