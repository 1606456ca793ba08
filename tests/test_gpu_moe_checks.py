"""Device-side checks of the grouped MoE GEMV's item list, and the per-row
combine when one output row receives many items.

An item's x_row outside the input rows reads zeros, an out_row outside y is not
written (accumulate == 0), and either sets the device status word to
SVQ_ERR_INVALID_ARG; nothing is read or written out of bounds.  With
accumulate == 1, each output row is the sum of its items in item order, also
for a row with more items than the combine kernel's shared list (2048)."""
import numpy as np
import pytest

import oracle
import synth
from tests.gpu_util import need_gpu, rel_err, torch, x_f16

import bit_spherical_vector_b200 as svq

pytestmark = pytest.mark.gpu
TOL = 1e-3


def _one_matrix(N=256, K=256, b_d=7):
    m = synth.make_matrix(96, 0, N, K, b_d)
    return m, svq.SvqWeight.from_synth(m)


def test_out_of_range_rows_are_reported_and_not_touched():
    need_gpu()
    m, W = _one_matrix()
    tab = svq.descriptor_table([W])
    x_bits = synth.make_x(96, 1, 2, m.K)
    x = x_f16(x_bits)
    # items: 0 valid, 1 x_row = 5 (x has 2 rows), 2 out_row = 7 (y has 3 rows), 3 valid
    mat = torch.zeros(4, dtype=torch.int32, device="cuda")
    xr = torch.tensor([0, 5, 1, 1], dtype=torch.int32, device="cuda")
    orow = torch.tensor([0, 1, 7, 2], dtype=torch.int32, device="cuda")
    items = svq.item_table(mat, xr, orow, torch.ones(4, device="cuda"))
    # y is a view inside a larger buffer filled with a sentinel, so a stray write would show
    big = torch.full((8, m.N), 12345.0, dtype=torch.float32, device="cuda")
    y = big[2:5]
    ws = torch.empty(max(svq.svq_moe_grouped_gemv_workspace_size(1, 4, m.N, False), 256), dtype=torch.uint8,
                     device="cuda")
    assert svq.svq_get_device_status() == svq.SVQ_OK
    svq.svq_moe_grouped_gemv(tab, 1, m.N, m.K, 8, items, 4, 4, x, svq.SVQ_X_F16, y, 3, False, ws)
    torch.cuda.synchronize()
    assert svq.svq_get_device_status() == svq.SVQ_ERR_INVALID_ARG
    yr, den = oracle.linear(m, x_bits)
    got = y.cpu().numpy()
    assert rel_err(got[0:1], yr[0:1], den[0:1]) <= TOL          # item 0
    assert rel_err(got[2:3], yr[1:2], den[1:2]) <= TOL          # item 3
    # item 1 (bad x_row) wrote zeros to row 1; item 2 (bad out_row) wrote nothing
    assert np.all(got[1] == 0.0)
    rest = torch.cat([big[:2], big[5:]]).cpu().numpy()
    assert np.all(rest == 12345.0)
    assert svq.svq_get_device_status() == svq.SVQ_OK              # the query clears the word


@pytest.mark.parametrize("n_items", [9, 2100])
def test_combine_many_items_one_row(n_items):
    """accumulate == 1 with every item on output row 1 (of 3), scales 1/(i+1): the row equals the sum of the
    items in item order (the 2100-item case exceeds the shared list and takes the fallback scan)."""
    need_gpu()
    m, W = _one_matrix(N=128, K=128, b_d=6)
    tab = svq.descriptor_table([W])
    T = 5
    x_bits = synth.make_x(97, 2, T, m.K)
    x = x_f16(x_bits)
    xr = torch.arange(n_items, device="cuda") % T
    scale = 1.0 / (torch.arange(n_items, device="cuda", dtype=torch.float32) + 1.0)
    items = svq.item_table(torch.zeros(n_items, dtype=torch.int32, device="cuda"), xr,
                           torch.ones(n_items, dtype=torch.int32, device="cuda"), scale)
    y = torch.full((3, m.N), -7.0, dtype=torch.float32, device="cuda")
    ws = torch.empty(svq.svq_moe_grouped_gemv_workspace_size(1, n_items, m.N, True), dtype=torch.uint8,
                     device="cuda")
    svq.svq_moe_grouped_gemv(tab, 1, m.N, m.K, 8, items, n_items, 4, x, svq.SVQ_X_F16, y, 3, True, ws)
    torch.cuda.synchronize()
    assert svq.svq_get_device_status() == svq.SVQ_OK
    yr, den = oracle.linear(m, x_bits)                              # [T][N]
    sc = scale.cpu().numpy().astype(np.float64)
    xi = xr.cpu().numpy()
    exp = np.zeros(m.N)
    dexp = np.zeros(m.N)
    for i in range(n_items):
        exp += sc[i] * yr[xi[i]]
        dexp += sc[i] * den[xi[i]]
    got = y.cpu().numpy()
    assert rel_err(got[1:2], exp[None], dexp[None]) <= TOL
    assert np.all(got[0] == -7.0) and np.all(got[2] == -7.0)      # rows without items untouched
