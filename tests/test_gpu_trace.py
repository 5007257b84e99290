"""Per-launch device timing (cf_trace_enable / cf_trace_read).

Every kernel a tracing context launches is bracketed by CUDA events; the
read-out lists each kernel with its launch count and summed time, and the
counts follow the call structure (two launches per quantised step, 5 products
and 4 CholeskyQR pairs and an apply per low-rank call at T = 2)."""
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def cf():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import activation_residual_compression_02_b200 as m

    m.lib()
    return m


def test_trace_quant_steps(cf):
    shapes = [(64, 512), (33, 256)]
    ctx = cf.Context(shapes, bits=2, group=128)
    st = cf.QuantState(shapes, 2, 128)
    xs = [torch.randn(r * c, device="cuda").to(torch.bfloat16) for r, c in shapes]
    ctx.trace(True)
    for t in range(3):
        sl = st.slots(xs)
        ctx.compress(sl, t)
        ctx.decompress(sl, t)
    got = {e["kernel"]: e for e in ctx.trace_read()}
    names = list(got)
    assert [n.split(",")[0] for n in names] == ["k_quant<op 0", "k_quant<op 1", "k_quant<op 2", "k_quant<op 3"]
    assert [got[n]["launches"] for n in names] == [1, 1, 2, 2]
    assert all(got[n]["total_ms"] > 0 for n in names)
    assert ctx.trace_read() == []                  # read-out clears
    ctx.trace(False)
    sl = st.slots(xs)
    ctx.compress(sl, 3)
    ctx.decompress(sl, 3)
    assert ctx.trace_read() == []                  # nothing traced while off
    assert ctx.check() == cf.CF_OK


def test_trace_lowrank_call(cf):
    m, n, r, T, k = 512, 768, 16, 2, 3
    ctx = cf.Context([], mode=cf.CF_MODE_LOWRANK, rank=r, iters=T)
    ws = torch.empty(ctx.lowrank_workspace_bytes(k, m, n), dtype=torch.uint8, device="cuda")
    ctx.set_workspace(ws)
    A = [synth.lowrank_matrix(m, n, r, mat=i).cuda() for i in range(k)]
    Q0 = [synth.q0(n, r, seed=0, mat=i).cuda() for i in range(k)]
    U = [torch.empty(m, r, device="cuda") for _ in A]
    R = [torch.empty(r, r, device="cuda") for _ in A]
    V = [torch.empty(n, r, device="cuda") for _ in A]
    E = [torch.empty(m, n, device="cuda") for _ in A]
    ctx.lowrank(A, Q0, U, R, V, E)                 # untraced first call
    ctx.trace(True)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    ctx.lowrank(A, Q0, U, R, V, E)
    e1.record()
    torch.cuda.synchronize()
    got = {e["kernel"]: e for e in ctx.trace_read()}
    want = {"k_cholqr_factor<Q>": T + 1, "k_cholqr_apply<Q>": T + 1, "k_gemm_tf32<16>": 2 * T + 1,
            "k_cholqr_factor<U>": 1, "k_cholqr_apply<U>": 1, "k_apply_async": 1}
    assert {n: e["launches"] for n, e in got.items()} == want
    traced = sum(e["total_ms"] for e in got.values())
    assert 0 < traced <= e0.elapsed_time(e1) * 1.01 + 0.05
    assert ctx.check() == cf.CF_OK
