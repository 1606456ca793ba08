"""GPU parity of the grouped MoE GEMV (device-side routing) against the CPU oracle.

Qwen3-30B-A3B-shaped MoE FFN: hidden 2048, 128 experts, moe_intermediate 768,
top-8 routing from softmax over seeded N(0,1) logits, renormalised.  Stage 1 is
one grouped call over all gate and up matrices; stage 2 one grouped call over
the down matrices with the fused fp16(silu(gate) * up) input and the routing
weights as out_scale, accumulated per token in item order.
Bar: 1e-3 of sum |W| |in| (GEMV tolerance) for every output."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import need_gpu, rel_err, torch, x_f16

import bit_spherical_vector_b200 as svq

pytestmark = pytest.mark.gpu
TOL = 1e-3


@pytest.fixture(scope="module")
def moe_setup():
    need_gpu()
    experts = synth.moe_experts()
    gu = []
    down = []
    for g, u, d in experts:
        gu += [svq.SvqWeight.from_synth(g), svq.SvqWeight.from_synth(u)]
        down.append(svq.SvqWeight.from_synth(d))
    torch.cuda.synchronize()
    return experts, gu, down


def _run_moe(gu, down, x_bits, ids, w):
    T, k = ids.shape
    dev = "cuda"
    ids_d = torch.from_numpy(ids.astype(np.int64)).to(dev)
    tok = torch.arange(T, device=dev).repeat_interleave(k)
    pair = torch.arange(T * k, device=dev)
    e = ids_d.reshape(-1)
    # stage 1: gate (matrix 2e) and up (2e + 1) of every (token, slot) pair
    items1 = svq.item_table(torch.stack([2 * e, 2 * e + 1], 1).reshape(-1), tok.repeat_interleave(2),
                            torch.stack([2 * pair, 2 * pair + 1], 1).reshape(-1),
                            torch.ones(2 * T * k, device=dev))
    gu_tab = svq.descriptor_table(gu)
    y1 = torch.empty((2 * T * k, 768), dtype=torch.float32, device=dev)
    ws1 = torch.empty(svq.svq_moe_grouped_gemv_workspace_size(len(gu), 2 * T * k, 768, False),
                      dtype=torch.uint8, device=dev)
    svq.svq_moe_grouped_gemv(gu_tab, len(gu), 768, 2048, 8, items1, 2 * T * k, T, x_f16(x_bits),
                             svq.SVQ_X_F16, y1, 2 * T * k, False, ws1)
    # stage 2: down of every pair, input silu(gate) * up from stage 1, weighted sum per token
    items2 = svq.item_table(e, pair, tok, torch.from_numpy(w.reshape(-1)).to(dev))
    dn_tab = svq.descriptor_table(down)
    out = torch.full((T, 2048), float("nan"), dtype=torch.float32, device=dev)
    ws2 = torch.empty(svq.svq_moe_grouped_gemv_workspace_size(len(down), T * k, 2048, True),
                      dtype=torch.uint8, device=dev)
    svq.svq_moe_grouped_gemv(dn_tab, len(down), 2048, 768, 8, items2, T * k, T, y1.view(T * k, 2 * 768),
                             svq.SVQ_X_SWIGLU_F32, out, T, True, ws2)
    torch.cuda.synchronize()
    assert svq.svq_get_device_status() == svq.SVQ_OK
    return y1.cpu().numpy().reshape(T, k, 2, 768), out.cpu().numpy()


@pytest.mark.parametrize("T", [1, 16])
def test_moe_ffn_against_oracle(moe_setup, T):
    experts, gu, down = moe_setup
    x = synth.moe_x(T)
    ids, w = synth.moe_routing(T)
    y1, out = _run_moe(gu, down, x, ids, w)
    # stage 1 (gate and up of every pair) against the oracle's layers
    for t in range(T):
        for s in range(ids.shape[1]):
            g, u, _ = experts[ids[t, s]]
            for which, m in ((0, g), (1, u)):
                y_ref, den = oracle.linear(m, x[t:t + 1])
                assert rel_err(y1[t, s, which][None], y_ref, den) <= TOL
    # stage 2: the oracle's FFN fed with this run's stage-1 activations, rounded to fp16 as the
    # kernel does (silu in fp64 here, fp32 there: an fp16 rounding of h may differ by one unit)
    h = oracle.silu(y1[:, :, 0].astype(np.float64)) * y1[:, :, 1]
    h_bits = oracle.f2h_rne(h.astype(np.float32)).reshape(h.shape)
    _, _, ref, den = oracle.moe_ffn(experts, x, ids, w, h_bits=h_bits)
    assert rel_err(out, ref, den) <= TOL + 2.0 ** -11


def test_moe_reproducible(moe_setup):
    experts, gu, down = moe_setup
    x = synth.moe_x(16)
    ids, w = synth.moe_routing(16)
    _, out1 = _run_moe(gu, down, x, ids, w)
    _, out2 = _run_moe(gu, down, x, ids, w)
    assert np.array_equal(out1, out2)


def test_moe_large_routing_table_stage1(moe_setup):
    """300 tokens x top-8: 4800 (matrix, token) items in the gate/up stage, more than the
    kernel builds in shared memory, so the routing goes through route_kernel and the
    workspace.  Sampled items against the oracle's single-matrix layer."""
    experts, gu, _ = moe_setup
    T = 300
    x = synth.moe_x(T)
    ids, _ = synth.moe_routing(T)
    k = ids.shape[1]
    dev = "cuda"
    e = torch.from_numpy(ids.astype(np.int64)).to(dev).reshape(-1)
    tok = torch.arange(T, device=dev).repeat_interleave(k)
    pair = torch.arange(T * k, device=dev)
    items = svq.item_table(torch.stack([2 * e, 2 * e + 1], 1).reshape(-1), tok.repeat_interleave(2),
                           torch.stack([2 * pair, 2 * pair + 1], 1).reshape(-1), torch.ones(2 * T * k, device=dev))
    y = torch.empty((2 * T * k, 768), dtype=torch.float32, device=dev)
    ws = torch.empty(svq.svq_moe_grouped_gemv_workspace_size(len(gu), 2 * T * k, 768, False),
                     dtype=torch.uint8, device=dev)
    counts = np.bincount(ids.reshape(-1), minlength=len(experts))
    svq.svq_moe_grouped_gemv(svq.descriptor_table(gu), len(gu), 768, 2048, 8, items, 2 * T * k,
                             int(counts.max()), x_f16(x), svq.SVQ_X_F16, y, 2 * T * k, False, ws)
    torch.cuda.synchronize()
    assert svq.svq_get_device_status() == svq.SVQ_OK
    y = y.cpu().numpy().reshape(T, k, 2, 768)
    rng = np.random.default_rng(7)
    for t in rng.choice(T, 12, replace=False):
        s = int(rng.integers(k))
        g, u, _ = experts[ids[t, s]]
        for which, m in ((0, g), (1, u)):
            y_ref, den = oracle.linear(m, x[t:t + 1])
            assert rel_err(y[t, s, which][None], y_ref, den) <= TOL
