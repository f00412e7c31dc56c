"""GPU parity of the c/g producer (dc_attn_cg_fwd, dc_attn_cg_bwd) against the fp64 oracle.

Tolerances come from the arithmetic: every output is a sum of products taken in fp32
(x converted exactly from bf16), so its error is at most gamma_n * sum |terms| with
gamma_n = n * 2^-24 / (1 - n * 2^-24) and n the longest chain of additions.  The
kernels' chains: forward at most D/16 + 8 terms per half of a column slice, the two
halves, 8 slices and the bias; dx 2H terms; dweight
and dbias the tokens of one partial record (ceil(N / blocks), blocks <= 148) in order,
then the records added in 16 strided sums and those 16 in order.  The oracle run on |x|, |w|, |e| gives sum |terms|.
A bf16 dx adds its own rounding, 2^-9 of the value.
"""
import numpy as np
import pytest
import torch

import oracle
from cross_head_dynamic_b200 import dcattn
from cross_head_dynamic_b200.inputs import cg_problem

pytestmark = pytest.mark.gpu

U = 2.0 ** -24


def gamma(n):
    return n * U / (1 - n * U)


@pytest.fixture(scope="module", autouse=True)
def _setup():
    oracle.build()
    dcattn.load_library()


def _to_np(t):
    return t.detach().double().cpu().numpy()


def _run(p, dtype, impl="auto", dx_impl=None):
    dev = "cuda"
    x = p["x"].to(dev)
    w = p["w"].to(dev).t().contiguous()      # weight [2H][D]
    b = p["b"].to(dev)
    dc, dg = p["dc"].to(dev), p["dg"].to(dev)
    c, g = dcattn.dc_attn_cg_fwd(x, w, b, impl=impl)
    dx, dw, db = dcattn.dc_attn_cg_bwd(x, w, dc, dg, impl=dx_impl or _dx_impl(p, impl))
    torch.cuda.synchronize()
    return c, g, dx, dw, db


def _dx_on_tc(p):
    """The conditions under which AUTO runs dx on tcgen05 (contiguous dx)."""
    N, D = p["x"].shape
    H = p["dc"].shape[1]
    return p["x"].dtype == torch.bfloat16 and 2 * H <= 16 and D % 8 == 0 and D <= 2048


def _dw_on_tc(p):
    """The conditions under which AUTO runs the dweight partial sums on tcgen05 (contiguous x)."""
    N, D = p["x"].shape
    H = p["dc"].shape[1]
    return p["x"].dtype == torch.bfloat16 and 2 * H <= 16 and D % 8 == 0 and N >= 64 and D >= 64


def _dx_impl(p, fwd_impl):
    """The backward's impl argument: AUTO (each kernel on tcgen05 where it can) unless the
    forward was asked to run SIMT."""
    return "simt" if fwd_impl == "simt" else "auto"


def _families(p, bwd_impl):
    """(dx family, dweight family) that a backward call with `bwd_impl` runs: AUTO takes
    tcgen05 for dx where possible and keeps dweight on the CUDA cores; TCGEN05 both."""
    if bwd_impl == "simt":
        return "simt", "simt"
    if bwd_impl == "tcgen05":
        return "tcgen05", "tcgen05"
    return ("tcgen05" if _dx_on_tc(p) else "simt"), "simt"


def _fwd_tolerance(D, fwd_impl):
    """Relative to the sum of |terms|.  SIMT: fp32 FMAs in the kernel's order.  tcgen05: the
    products with the bf16 weight terms are exact and the terms sum to the weight within
    2^-24; the tensor core's fp32 accumulation is not specified to round to nearest, so each
    of its ceil(D/16) accumulation steps is allowed 2 units in the last place (2^-22) of the
    sum of |terms|, plus the epilogue's three additions and the bias."""
    if fwd_impl == "simt":
        return gamma(D // 16 + 18)
    return (-(-D // 16) + 2) * 2.0 ** -22 + 2.0 ** -24 + gamma(4)


def _dx_tolerance(H, dx_impl):
    """Relative to the sum of |terms|, before the bf16 rounding of dx.  SIMT: 2H fp32 FMAs
    in order.  tcgen05: six of the nine products of the bf16 splits of e and the weight,
    2^-23 of |e w| left out, accumulated by the tensor core in 6 steps of 16 (2^-22 each)."""
    if dx_impl == "simt":
        return gamma(2 * H + 2)
    return 8 * 2.0 ** -22 + 2.0 ** -23


def _dw_tolerance(N, blocks, dw_impl):
    """dweight, relative to the sum of |terms|.  SIMT: the tokens of one record in two
    interleaved halves (even and odd tokens), each in order, the halves added, then the
    records (16 strided sums, then those 16); bounded by the sum of one record's tokens in
    order.  tcgen05: exact products of x with the bf16
    splits of e (2^-24 left out), the tensor core's accumulation over ceil(span / 16) steps,
    the epilogue's two additions, then the same record sums."""
    span = -(-N // blocks)
    reduce = gamma(blocks // 16 + 18)
    if dw_impl == "simt":
        return gamma(span + blocks // 16 + 18)
    return (-(-span // 16) + 2) * 2.0 ** -22 + 2.0 ** -24 + gamma(2) + reduce


def _db_tolerance(N, blocks, dw_impl):
    """dbias.  SIMT: twelve interleaved parts of one record's tokens, each in order, then the
    twelve and the records; bounded by the sum of the record's tokens in order."""
    span = -(-N // blocks)
    if dw_impl == "simt":
        return gamma(span + blocks // 16 + 18)
    return gamma(span // 64 + 66 + blocks // 16 + 18)   # 64 strided sums, then those 64, then the records


def _check(p, outs, dtype, fwd_impl="simt", dx_impl=None):
    c, g, dx, dw, db = (_to_np(t) for t in outs)
    x, w, b = _to_np(p["x"]), _to_np(p["w"]), _to_np(p["b"])
    dcn, dgn = _to_np(p["dc"]), _to_np(p["dg"])
    N, D = x.shape
    H = dcn.shape[1]
    rc, rg = oracle.cg_forward(x, w, b)
    mc, mg = oracle.cg_forward(np.abs(x), np.abs(w), np.abs(b))
    tf = _fwd_tolerance(D, fwd_impl)
    assert np.all(np.abs(c - rc) <= tf * mc + 1e-30), np.abs(c - rc).max()
    assert np.all(np.abs(g - rg) <= tf * mg + 1e-30), np.abs(g - rg).max()
    rdx, rdw, rdb = oracle.cg_backward(x, w, dcn, dgn)
    mdx, mdw, mdb = oracle.cg_backward(np.abs(x), np.abs(w), np.abs(dcn), np.abs(dgn))
    dx_fam, dw_fam = _families(p, dx_impl or _dx_impl(p, fwd_impl))
    tol_dx = _dx_tolerance(H, dx_fam) * mdx + (2.0 ** -8 * np.abs(rdx) if dtype == "bf16" else 0) + 1e-30
    assert np.all(np.abs(dx - rdx) <= tol_dx), np.abs(dx - rdx).max()
    blocks = min(max((N + 63) // 64, 1), 148)
    tw, tb = _dw_tolerance(N, blocks, dw_fam), _db_tolerance(N, blocks, dw_fam)
    assert np.all(np.abs(dw.T - rdw) <= tw * mdw + 1e-30), np.abs(dw.T - rdw).max()
    assert np.all(np.abs(db - rdb) <= tb * mdb + 1e-30), np.abs(db - rdb).max()


@pytest.mark.parametrize("N, D, H, dtype", [
    (4096, 768, 6, "bf16"),      # GPT-2 small width, several blocks and a full grid
    (1000, 768, 6, "f32"),
    (333, 64, 1, "bf16"),        # 2H = 2 padded to 8, D below one 64-element pass
    (77, 130, 3, "f32"),         # ragged D (not a multiple of 64), ragged N
    (517, 256, 16, "bf16"),      # 2H = 32, two tokens per warp
    (129, 512, 12, "bf16"),      # 2H = 24
    (640, 96, 8, "f32"),         # 2H = 16
    (5, 2, 4, "bf16"),           # D = 2: one pair, most lanes idle
    (1, 768, 6, "bf16"),         # one token
    (65, 768, 5, "bf16"),        # 2H = 10 padded to 12; one record boundary crossed
])
def test_cg_parity(N, D, H, dtype):
    p = cg_problem(100 + N + D + H, N, D, H, dtype)
    impls = ["simt"]
    if dcattn.dc_attn_cg_resolve_impl(p["x"].cuda(), H) == "tcgen05":
        impls.append("tcgen05")
    for impl in impls:
        _check(p, _run(p, dtype, impl), dtype, impl)


@pytest.mark.parametrize("N, D, H", [
    (128, 64, 1),        # one tile, one 64-column block
    (300, 200, 6),       # ragged tile and a ragged column block (zero-filled by TMA)
    (1000, 2048, 8),     # widest weight that fits at 2H = 16 (a 2-stage x ring)
    (777, 1024, 16),     # 32 outputs per split, widest that fits
    (513, 768, 16),      # 32 outputs per split, a 5-stage ring
    (4099, 768, 6),      # GPT-2 width, ragged last tile
    (256, 768, 3),       # 2H = 6 padded to 16 per split
])
def test_cg_forward_tcgen05(N, D, H):
    p = cg_problem(200 + N + D + H, N, D, H, "bf16")
    assert dcattn.dc_attn_cg_resolve_impl(p["x"].cuda(), H) == "tcgen05"
    _check(p, _run(p, "bf16", "tcgen05"), "bf16", "tcgen05")


@pytest.mark.parametrize("N, D, H", [
    (128, 64, 1),        # one tile, one 64-column chunk
    (300, 200, 6),       # ragged tile, D not a multiple of 16 (last columns stored singly)
    (1000, 1024, 8),     # four 256-column chunks
    (600, 2048, 8),      # widest weight that fits, eight chunks
    (4099, 768, 6),      # GPT-2 width, three chunks alternating the two TMEM buffers
    (65, 328, 4),        # fewer tokens than a tile; a 64-column last chunk (5 blocks)
])
def test_cg_backward_tcgen05(N, D, H):
    """dx and the dweight partial sums both on tcgen05 (forced)."""
    p = cg_problem(300 + N + D + H, N, D, H, "bf16")
    _check(p, _run(p, "bf16", "simt", "tcgen05"), "bf16", "simt", "tcgen05")


@pytest.mark.parametrize("N, D, H, dtype", [
    (100000, 256, 6, "bf16"),    # 676 tokens per record: the 4-stage ring of 64-token stages wraps
    (30001, 768, 6, "bf16"),     # 203 tokens per record at the GPT-2 width, ragged last stage
    (20000, 1030, 4, "f32"),     # fp32 x, D % 4 == 2, two passes over the columns
    (9000, 520, 16, "bf16"),     # 2H = 32 (one column pair per thread), two passes
])
def test_cg_dweight_simt_spans(N, D, H, dtype):
    """The CUDA-core dweight on long token ranges per record (many stages through the ring)."""
    p = cg_problem(500 + N + D + H, N, D, H, dtype)
    _check(p, _run(p, dtype, "simt"), dtype, "simt")


@pytest.mark.parametrize("N", [64, 8191, 20000, 300000])
def test_cg_dweight_tcgen05_spans(N):
    """Token ranges of 1, several and many 64-token chunks per record (the record count is
    capped at 148), a ragged last chunk, and ranges that end inside a TMA box."""
    p = cg_problem(400 + N, N, 256, 6, "bf16")
    assert _dw_on_tc(p)
    _check(p, _run(p, "bf16", "simt", "tcgen05"), "bf16", "simt", "tcgen05")


def test_cg_gpt2_full_size():
    """The GPT-2 training shape: 16384 tokens (8 x 2048), D = 768, H = 6, every output, on
    both forward families."""
    p = cg_problem(7, 16384, 768, 6, "bf16")
    for impl in ("simt", "tcgen05"):
        _check(p, _run(p, "bf16", impl), "bf16", impl)


def test_cg_backward_is_deterministic():
    p = cg_problem(8, 20000, 768, 6, "bf16")
    a = _run(p, "bf16")
    b = _run(p, "bf16")
    for u, v in zip(a, b):
        assert torch.equal(u, v)


def test_cg_zero_tokens_writes_zero_gradients():
    dev = "cuda"
    x = torch.empty(0, 64, device=dev, dtype=torch.bfloat16)
    w = torch.randn(8, 64, device=dev)
    dw = torch.full((8, 64), 7.0, device=dev)
    db = torch.full((8,), 7.0, device=dev)
    e = torch.empty(0, 4, device=dev)
    c, g = dcattn.dc_attn_cg_fwd(x, w, torch.zeros(8, device=dev))
    assert c.shape == (0, 4)
    dx, dw, db = dcattn.dc_attn_cg_bwd(x, w, e, e, dweight=dw, dbias=db)
    torch.cuda.synchronize()
    assert not dw.any() and not db.any()


@pytest.mark.parametrize("width, impl", [(266, "simt"), (264, "tcgen05")])
def test_cg_strided_rows(width, impl):
    """x a column slice of a wider hidden-state buffer, dx written into a wider buffer:
    results equal those of contiguous tensors on the same kernel families, and the gap
    columns stay untouched.  Rows 532 bytes apart (no TMA): SIMT; 528 bytes apart: every
    kernel on tcgen05."""
    p = cg_problem(9, 700, 256, 6, "bf16")
    dev = "cuda"
    base = torch.randn(700, width, device=dev).to(torch.bfloat16)
    base[:, 8:264] = p["x"].to(dev)          # 16-byte aligned start
    xs = base[:, 8:264]
    w = p["w"].to(dev).t().contiguous()
    b = p["b"].to(dev)
    dc, dg = p["dc"].to(dev), p["dg"].to(dev)
    dxbuf = torch.full((700, 256 + 16), 3.0, device=dev, dtype=torch.bfloat16)
    assert dcattn.dc_attn_cg_resolve_impl(xs, 6) == ("simt" if width == 266 else "tcgen05")
    c, g = dcattn.dc_attn_cg_fwd(xs, w, b, impl=impl)
    dx, dw, db = dcattn.dc_attn_cg_bwd(xs, w, dc, dg, dx=dxbuf[:, 8:264], impl=impl)
    ref = _run(p, "bf16", impl, impl)
    torch.cuda.synchronize()
    for u, v in zip((c, g, dxbuf[:, 8:264], dw, db), ref):
        assert torch.equal(u, v)
    assert bool((dxbuf[:, :8] == 3).all()) and bool((dxbuf[:, 264:] == 3).all())


def test_cg_feeds_the_attention_forward():
    """x -> (c, g) -> windowed attention, against the oracle chain in fp64."""
    N, D, H, d, W = 600, 256, 4, 64, 112
    p = cg_problem(10, N, D, H, "bf16")
    dev = "cuda"
    gen = torch.Generator().manual_seed(11)
    q, k, v = (torch.randn(N, H, d, generator=gen).to(torch.bfloat16) for _ in range(3))
    cu = torch.tensor([0, 250, 600], dtype=torch.int32)
    c, g = dcattn.dc_attn_cg_fwd(p["x"].to(dev), p["w"].to(dev).t().contiguous(), p["b"].to(dev))
    scale = d ** -0.5
    o, _, _ = dcattn.dc_attn_fwd(q.to(dev), k.to(dev), v.to(dev), c, g, cu.to(dev), W, scale)
    torch.cuda.synchronize()
    rc, rg = oracle.cg_forward(_to_np(p["x"]), _to_np(p["w"]), _to_np(p["b"]))
    ro = oracle.forward(_to_np(q), _to_np(k), _to_np(v), rc, rg, cu.numpy(), W, scale)[0]
    err = np.abs(_to_np(o) - ro)
    assert err.max() <= 0.02 * np.abs(ro).max(), err.max()


@pytest.mark.parametrize("N, D, H", [(16384, 768, 6), (300, 200, 6), (777, 1024, 16), (256, 64, 1)])
def test_cg_prepared_weight_is_bit_identical(N, D, H):
    """The tensor-core kernels give the same bits whether they convert the weight themselves
    or copy the image dc_attn_cg_prepare wrote (H = 16: the forward's image only; dx then
    runs on the CUDA cores and ignores it)."""
    p = cg_problem(500 + N + D + H, N, D, H, "bf16")
    dev = "cuda"
    x, w, b = p["x"].to(dev), p["w"].to(dev).t().contiguous(), p["b"].to(dev)
    dc, dg = p["dc"].to(dev), p["dg"].to(dev)
    img = dcattn.dc_attn_cg_prepare(w)
    for use in (None, img):
        outs = dcattn.dc_attn_cg_fwd(x, w, b, weight_splits=use) + dcattn.dc_attn_cg_bwd(x, w, dc, dg,
                                                                                        weight_splits=use)
        torch.cuda.synchronize()
        if use is None:
            ref = [t.clone() for t in outs]
    for u, v in zip(outs, ref):
        assert torch.equal(u, v)
    _check(p, outs, "bf16", "auto")


def test_cg_chain_backward_through_the_attention():
    """The whole layer chain on the GPU, x -> (c, g) -> windowed attention -> backward ->
    (dc, dg) -> dx, dweight, dbias, against the same chain in the fp64 oracle (bf16
    attention: compared relative to each output's largest magnitude)."""
    N, D, H, d, W = 700, 256, 6, 128, 112
    p = cg_problem(12, N, D, H, "bf16")
    dev = "cuda"
    gen = torch.Generator().manual_seed(13)
    q, k, v, dO = (torch.randn(N, H, d, generator=gen).to(torch.bfloat16) for _ in range(4))
    cu = torch.tensor([0, 300, 700], dtype=torch.int32)
    scale = d ** -0.5
    x, w, b = p["x"].to(dev), p["w"].to(dev).t().contiguous(), p["b"].to(dev)
    img = dcattn.dc_attn_cg_prepare(w)
    c, g = dcattn.dc_attn_cg_fwd(x, w, b, weight_splits=img)
    qd, kd, vd, dOd, cud = q.to(dev), k.to(dev), v.to(dev), dO.to(dev), cu.to(dev)
    o, lse, pmap = dcattn.dc_attn_fwd(qd, kd, vd, c, g, cud, W, scale)
    dq, dk, dv, dcv, dgv = dcattn.dc_attn_bwd(qd, kd, vd, c, g, dOd, lse, pmap, cud, W, scale)
    dx, dw, db = dcattn.dc_attn_cg_bwd(x, w, dcv, dgv, weight_splits=img)
    torch.cuda.synchronize()
    rc, rg = oracle.cg_forward(_to_np(p["x"]), _to_np(p["w"]), _to_np(p["b"]))
    ro = oracle.forward(_to_np(q), _to_np(k), _to_np(v), rc, rg, cu.numpy(), W, scale)[0]
    rgrads = oracle.backward(_to_np(q), _to_np(k), _to_np(v), rc, rg, _to_np(dO), cu.numpy(), W, scale)
    rdx, rdw, rdb = oracle.cg_backward(_to_np(p["x"]), _to_np(p["w"]), rgrads[3], rgrads[4])
    for name, got, ref in (("o", o, ro), ("dq", dq, rgrads[0]), ("dc", dcv, rgrads[3]), ("dg", dgv, rgrads[4]),
                           ("dx", dx, rdx), ("dweight", dw.t(), rdw), ("dbias", db, rdb)):
        err = np.abs(_to_np(got) - ref).max() / np.abs(ref).max()
        assert err <= 2e-2, (name, err)
