"""GPU parity of nvfp4_amax / nvfp4_quantize (row-wise and column-wise, both scale layouts)
against the CPU oracle: codes, scales and g must match bit for bit, padding included.
Shapes span several tiles with ragged tails, the degenerate cases (zero tensor, one row, a
partial 16-block, tiny magnitudes where 1/d overflows, inf/NaN input) and the full-size tensors
of the DiT workloads."""
import numpy as np
import pytest
import torch

import bit_kv_cache_24_b200 as nv
from bit_kv_cache_24_b200 import synth
from tests.parity_util import assert_quantized_equal

pytestmark = pytest.mark.gpu

ROW_CASES = [(1, 16, "normal"), (3, 32, "outliers"), (128, 256, "outliers"), (130, 80, "wide"),
             (257, 3072, "lognormal"), (1000, 1008, "wide"), (4680, 3072, "lognormal")]
COL_CASES = [(16, 32, "normal"), (40, 24, "outliers"), (37, 8, "wide"), (300, 96, "lognormal"),
             (4680, 256, "wide"), (1040, 136, "normal")]


@pytest.mark.parametrize("layout", [nv.SF_LINEAR, nv.SF_MMA])
@pytest.mark.parametrize("rows,cols,kind", ROW_CASES)
def test_rowwise(orc, rows, cols, kind, layout):
    x = synth.ragged(rows + cols, rows, cols, kind)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gq = nv.nvfp4_quantize(x.cuda(), nv.ROWWISE, sf_layout=layout, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    ost, oq = orc.quantize(x)
    assert ost == 0
    assert_quantized_equal(orc, gq, oq, f"row {rows}x{cols} {kind}")


@pytest.mark.parametrize("layout", [nv.SF_LINEAR, nv.SF_MMA])
@pytest.mark.parametrize("rows,cols,kind", COL_CASES)
def test_colwise(orc, rows, cols, kind, layout):
    x = synth.ragged(rows * 3 + cols, rows, cols, kind)
    gq = nv.nvfp4_quantize(x.cuda(), nv.COLWISE, sf_layout=layout)
    ost, oq = orc.quantize(x, colwise=True)
    assert ost == 0
    assert_quantized_equal(orc, gq, oq, f"col {rows}x{cols} {kind}")


def test_strided_rows_and_amax_in(orc):
    big = synth.ragged(5, 300, 1024, "lognormal")
    x = big.cuda()[:, 128:640]                          # ld = 1024, K = 512
    amax = nv.nvfp4_amax(x)
    ref_st, ref_amax = orc.amax(big[:, 128:640].contiguous())
    assert amax.item() == np.float32(ref_amax)
    g1 = nv.nvfp4_quantize(x, nv.ROWWISE)
    g2 = nv.nvfp4_quantize(x, nv.ROWWISE, amax_in=amax)
    g3 = nv.nvfp4_quantize(x, nv.COLWISE, amax_in=amax)
    _, o1 = orc.quantize(big[:, 128:640].contiguous())
    _, o3 = orc.quantize(big[:, 128:640].contiguous(), colwise=True)
    assert_quantized_equal(orc, g1, o1, "strided")
    assert_quantized_equal(orc, g2, o1, "amax_in")
    assert_quantized_equal(orc, g3, o3, "colwise amax_in")


def test_zero_tensor(orc):
    x = torch.zeros(64, 96, dtype=torch.bfloat16)
    gq = nv.nvfp4_quantize(x.cuda(), nv.ROWWISE)
    _, oq = orc.quantize(x)
    assert_quantized_equal(orc, gq, oq, "zeros")
    assert gq.g.item() == 1.0


def test_tiny_magnitudes_where_reciprocal_overflows(orc):
    # BF16 subnormal-range inputs: g and d are so small that 1/d overflows to inf; the zero
    # elements then encode as +0 (their product would be NaN)
    a = np.zeros((4, 64), np.float32)
    a[0, :8] = 1e-39
    a[1, 3] = -3e-40
    a[2, ::3] = 2e-38
    a[3, 1] = 1e-30
    x = torch.from_numpy(a).to(torch.bfloat16)
    gq = nv.nvfp4_quantize(x.cuda(), nv.ROWWISE, sf_layout=nv.SF_LINEAR)
    _, oq = orc.quantize(x)
    assert_quantized_equal(orc, gq, oq, "tiny")


@pytest.mark.parametrize("bad", [float("inf"), float("nan")])
def test_nonfinite_input_sets_status(bad):
    x = torch.randn(64, 64).to(torch.bfloat16)
    x[17, 5] = bad
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    nv.nvfp4_quantize(x.cuda(), nv.ROWWISE, status=st)
    torch.cuda.synchronize()
    assert st.item() == nv.NVFP4_ERR_NONFINITE
    st.zero_()
    nv.nvfp4_quantize(x.cuda(), nv.COLWISE, status=st)
    torch.cuda.synchronize()
    assert st.item() == nv.NVFP4_ERR_NONFINITE


def test_full_size_training_operands(orc):
    """Training workload at full size: X [37440 x 3072] row-wise and column-wise (the wgrad
    operand), every byte compared."""
    X = synth.train()["X"]
    xg = X.cuda()
    amax = nv.nvfp4_amax(xg)
    gr = nv.nvfp4_quantize(xg, nv.ROWWISE, amax_in=amax)
    gc = nv.nvfp4_quantize(xg, nv.COLWISE, amax_in=amax)
    _, orow = orc.quantize(X)
    assert_quantized_equal(orc, gr, orow, "train X row")
    del orow
    _, ocol = orc.quantize(X, colwise=True)
    assert_quantized_equal(orc, gc, ocol, "train X col")


def test_full_size_ffn_down_activation(orc):
    A = synth.ffn()["A_down"]                           # GELU output [4680 x 14336]
    gq = nv.nvfp4_quantize(A.cuda(), nv.ROWWISE)
    _, oq = orc.quantize(A)
    assert_quantized_equal(orc, gq, oq, "ffn down A")


@pytest.mark.parametrize("rows,cols,kind", [(1, 16, "normal"), (37, 48, "outliers"), (300, 96, "wide"),
                                            (1040, 512, "lognormal"), (4680, 3072, "lognormal"), (6000, 256, "normal"),
                                            # cols % 64 == 0: the single-read kernel, ragged rows, row-wise
                                            # padding rows beyond the column layout's padded range
                                            (1, 64, "normal"), (17, 128, "outliers"), (129, 64, "wide"),
                                            (200, 192, "lognormal"), (2049, 320, "outliers")])
@pytest.mark.parametrize("layout", [nv.SF_LINEAR, nv.SF_MMA])
def test_rowcol_from_one_read(orc, rows, cols, kind, layout):
    """NVFP4_ROWCOL: row-wise and column-wise outputs of one call equal the oracle's, byte for byte
    (for cols % 64 == 0 from one kernel that reads x once, otherwise a row pass and a column pass)."""
    x = synth.ragged(rows * 5 + cols, rows, cols, kind)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gr, gc = nv.nvfp4_quantize(x.cuda(), nv.ROWCOL, sf_layout=layout, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    _, orow = orc.quantize(x)
    _, ocol = orc.quantize(x, colwise=True)
    assert_quantized_equal(orc, gr, orow, f"rowcol-row {rows}x{cols}")
    assert_quantized_equal(orc, gc, ocol, f"rowcol-col {rows}x{cols}")


def test_repeated_calls_share_workspace(orc):
    """Consecutive quantizations reuse one workspace: each call's amax partials and scale record
    overwrite the previous call's, and no result may depend on what the workspace held before."""
    L = nv.lib()
    ws = torch.empty(L.nvfp4_quantize_workspace(4680, 3072), dtype=torch.uint8, device="cuda")
    xs = [synth.ragged(40 + i, 4680, 3072, kind) for i, kind in enumerate(["lognormal", "wide", "normal"])]
    outs = [nv.nvfp4_quantize(x.cuda(), nv.ROWWISE, ws=ws) for x in xs]
    for x, g in zip(xs, outs):
        _, o = orc.quantize(x)
        assert_quantized_equal(orc, g, o, "shared ws")


@pytest.mark.parametrize("rows,cols,kind", [(37, 48, "outliers"), (300, 96, "wide"), (4680, 3072, "lognormal")])
@pytest.mark.parametrize("layout", [nv.SF_LINEAR, nv.SF_MMA])
def test_amax_given_builds_its_record_in_the_pass(orc, rows, cols, kind, layout):
    """With amax_in the quantize passes build the per-tensor scale record themselves (one launch
    per layout, no record kernel): row-wise, column-wise and both-layouts outputs and g equal the
    oracle's quantization with the same amax, byte for byte."""
    x = synth.ragged(rows * 3 + cols, rows, cols, kind)
    xg = x.cuda()
    amax = nv.nvfp4_amax(xg)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    gr = nv.nvfp4_quantize(xg, nv.ROWWISE, amax_in=amax, sf_layout=layout, status=st)
    gc = nv.nvfp4_quantize(xg, nv.COLWISE, amax_in=amax, sf_layout=layout, status=st)
    br, bc = nv.nvfp4_quantize(xg, nv.ROWCOL, amax_in=amax, sf_layout=layout, status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    a = np.float32(amax.item())
    _, orow = orc.quantize(x, amax_in=a)
    _, ocol = orc.quantize(x, colwise=True, amax_in=a)
    for got, want, label in ((gr, orow, "row"), (gc, ocol, "col"), (br, orow, "rowcol-row"), (bc, ocol, "rowcol-col")):
        assert_quantized_equal(orc, got, want, f"amax given {label} {rows}x{cols}")


@pytest.mark.parametrize("direction", [nv.ROWWISE, nv.COLWISE, nv.ROWCOL])
def test_nonfinite_amax_in_sets_status_and_writes_nothing(direction):
    x = synth.ragged(9, 64, 96, "normal").cuda()
    for bad in (float("inf"), float("nan")):
        amax = torch.tensor([bad], dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        outs = nv.nvfp4_quantize(x, direction, amax_in=amax, status=st)
        outs = outs if isinstance(outs, tuple) else (outs,)
        for q in outs:
            q.codes.fill_(0xAB)
            q.sf.fill_(0xCD)
            q.g.fill_(-1.0)
        torch.cuda.synchronize()
        nv.nvfp4_quantize(x, direction, amax_in=amax, status=st,
                          out=outs if direction == nv.ROWCOL else outs[0])
        torch.cuda.synchronize()
        assert st.item() == nv.NVFP4_ERR_NONFINITE
        for q in outs:
            assert bool((q.codes == 0xAB).all()) and bool((q.sf == 0xCD).all()) and q.g.item() == -1.0


@pytest.mark.parametrize("rows,cols", [(129, 64), (4680, 3072), (33, 192)])
def test_rowcol_mixed_scale_layouts(orc, rows, cols):
    """Both layouts from one call with different scale layouts for the two outputs (tensor-core
    layout row-wise, linear column-wise, and the reverse)."""
    x = synth.ragged(rows + 7 * cols, rows, cols, "lognormal")
    _, orow = orc.quantize(x)
    _, ocol = orc.quantize(x, colwise=True)
    for lr, lc in ((nv.SF_MMA, nv.SF_LINEAR), (nv.SF_LINEAR, nv.SF_MMA)):
        out = (nv.QTensor(rows, cols, lr), nv.QTensor(cols, rows, lc))
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        nv.nvfp4_quantize(x.cuda(), nv.ROWCOL, out=out, status=st)
        torch.cuda.synchronize()
        assert st.item() == 0
        assert_quantized_equal(orc, out[0], orow, f"mixed row {lr}")
        assert_quantized_equal(orc, out[1], ocol, f"mixed col {lc}")
