"""Host-side argument checks of every C-ABI entry point, table-driven, on a machine without a GPU.

For each export a baseline call with well-formed (fake, never dereferenced) device addresses must
get through every host check and fail only at its first CUDA step (there is no device here). Each
case then breaks exactly one argument and expects the status the header gives for it, returned
before anything reaches CUDA. Whether a call reached CUDA is read from hstu_last_cuda_error(),
which only CUDA failures set: before each call it is set to a known value by a call that fails at
a known CUDA step, and a host rejection leaves that value in place. Two such values are used
(35 from a kernel launch, 1 from a tensor-map encoding), so that a call whose own CUDA failure
gives one of them is still seen to change the other.

The addresses are fake, so the module runs only where no GPU is visible: on a GPU machine a check
that failed to reject a case would hand the fake address to a kernel.
"""
import ctypes
import math

import pytest
import torch

from hstu_sequential_transduction_causal_b200 import hstu as Hb

pytestmark = pytest.mark.skipif(torch.cuda.is_available(), reason="fake device addresses: CPU-only machine")

OK, INVALID, UNSUPPORTED, WORKSPACE, CUDA = 0, 1, 2, 3, 4
F32, BF16, F16 = Hb.HSTU_F32, Hb.HSTU_BF16, Hb.HSTU_F16


def fake(i: int) -> int:
    """A distinct, 256-byte aligned address that is never dereferenced."""
    return (i + 1) << 24


@pytest.fixture(scope="module")
def L():
    from hstu_sequential_transduction_causal_b200 import build
    build.build()
    Hb._lib = None
    return Hb.lib()


# Batches whose causal tile-pair bound exceeds the tile kernels' 32-bit row coordinates: 200M tokens at
# max_len 8192 (51M pairs, beyond 2^31 / 128 for the forward), and 40M tokens (10M pairs: within the
# forward's bound, beyond 2^31 / (H 128) for the backward with H = 2).
HUGE_FWD = dict(T=200_000_000, max_len=8192)
HUGE_BWD = dict(T=40_000_000, max_len=8192)


def jag(B=2, T=300, max_len=200, **kw):
    j = Hb.hstu_jagged_t(B=B, max_len=max_len, T=T, offsets=fake(0), timestamps=fake(1))
    for k, v in kw.items():
        setattr(j, k, v)
    return j


def _mark_launch(L):
    """Leaves a kernel launch's CUDA failure as the last CUDA error."""
    assert L.hstu_debug_timeout_probe(fake(0), 256, None) == CUDA
    return L.hstu_last_cuda_error()


def _mark_encode(L):
    """Leaves a tensor-map encoding failure (no driver here) as the last CUDA error."""
    L.hstu_uvqk_fwd(300, 256, BF16, F16, fake(2), 256, fake(3), fake(4), fake(5), fake(6), fake(7), 256, None)
    return L.hstu_last_cuda_error()


def attempt(L, call, **ov):
    """(status, reached_cuda) of call(**ov)."""
    m1 = _mark_launch(L)
    r1 = call(**ov)
    e1 = L.hstu_last_cuda_error()
    m2 = _mark_encode(L)
    r2 = call(**ov)
    e2 = L.hstu_last_cuda_error()
    assert m1 != m2 and r1 == r2
    return r1, (e1 != m1 or e2 != m2)


def passes_host_checks(L, call, **ov):
    r, reached = attempt(L, call, **ov)
    return reached and r != OK


def run_cases(L, call, cases):
    """call(**overrides) -> status. cases: (name, overrides, expected status)."""
    assert passes_host_checks(L, call), "the baseline call must pass every host check"
    bad = []
    for name, ov, want in cases:
        got, reached = attempt(L, call, **ov)
        if got != want or reached:
            bad.append(f"{name}: got {Hb.STATUS.get(got, got)}{' after reaching CUDA' if reached else ''}, "
                       f"expected {Hb.STATUS[want]} from the host")
    assert not bad, "\n".join(bad)


# ------------------------------------------------------------------------------------------------
def test_jagged_worklist(L):
    def call(j=None, items=fake(2), count=fake(3)):
        return L.hstu_jagged_worklist(ctypes.byref(j if j is not None else jag()), items, count, None)
    run_cases(L, call, [
        ("negative B", dict(j=jag(B=-1)), INVALID),
        ("negative T", dict(j=jag(T=-1)), INVALID),
        ("negative max_len", dict(j=jag(max_len=-1)), INVALID),
        ("no offsets", dict(j=jag(offsets=None)), INVALID),
        ("tokens without timestamps", dict(j=jag(timestamps=None)), INVALID),
        ("T beyond int32 rows", dict(j=jag(T=1 << 31)), UNSUPPORTED),
        ("no items", dict(items=None), INVALID),
        ("no count", dict(count=None), INVALID),
    ])
    assert L.hstu_worklist_capacity(ctypes.byref(jag(B=-1))) == -1
    assert L.hstu_worklist_capacity(ctypes.byref(jag(B=2, T=300))) == 2 + math.ceil(300 / 128)


def test_time_buckets(L):
    def call(nb=128, sq=fake(2), out=fake(3), j=None):
        return L.hstu_time_buckets(ctypes.byref(j if j is not None else jag()), nb, sq, out, None)
    run_cases(L, call, [
        ("zero buckets", dict(nb=0), UNSUPPORTED),
        ("129 buckets", dict(nb=129), UNSUPPORTED),
        ("no square offsets", dict(sq=None), INVALID),
        ("no output", dict(out=None), INVALID),
        ("no offsets", dict(j=jag(offsets=None)), INVALID),
    ])


def test_uvqk_fwd(L):
    def call(T=300, D=256, dt=BF16, act=F16, x=fake(2), ld_x=256, W1=fake(3), b1=fake(4), uvqk=fake(5), z=fake(6),
             ws=fake(7), ws_bytes=256):
        return L.hstu_uvqk_fwd(T, D, dt, act, x, ld_x, W1, b1, uvqk, z, ws, ws_bytes, None)
    run_cases(L, call, [
        ("negative T", dict(T=-1), INVALID),
        ("D not a multiple of 64 (BF16)", dict(D=100, ld_x=104), UNSUPPORTED),
        ("F16 compute dtype", dict(dt=F16), UNSUPPORTED),
        ("F32 activations with BF16 operands", dict(act=F32), UNSUPPORTED),
        ("F16 activations with F32 operands", dict(dt=F32), UNSUPPORTED),
        ("no workspace", dict(ws=None), INVALID),
        ("workspace below 256 bytes", dict(ws_bytes=255), WORKSPACE),
        ("no x", dict(x=None), INVALID),
        ("no W1", dict(W1=None), INVALID),
        ("no output", dict(uvqk=None), INVALID),
        ("ld_x below D", dict(ld_x=248), INVALID),
        ("ld_x not a multiple of 8", dict(ld_x=260), UNSUPPORTED),
        ("x off 16 bytes", dict(x=fake(2) + 8), UNSUPPORTED),
        ("W1 off 16 bytes", dict(W1=fake(3) + 2), UNSUPPORTED),
        ("b1 off 16 bytes", dict(b1=fake(4) + 4), UNSUPPORTED),
        ("z off 16 bytes", dict(z=fake(6) + 2), UNSUPPORTED),
    ])
    assert attempt(L, call, T=0) == (OK, False)   # nothing to do, nothing enqueued
    assert passes_host_checks(L, call, b1=None) and passes_host_checks(L, call, z=None)   # both optional


def attn_desc(**kw):
    d = Hb.make_attn_desc(2, 64, 64, 1.0 / 256, 256, BF16, 1024, 1024, 1024, 128)
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_attn_fwd(L):
    need = L.hstu_attn_workspace_size(ctypes.byref(attn_desc()), ctypes.byref(jag()))
    assert need > 256
    assert L.hstu_attn_workspace_size(ctypes.byref(attn_desc()), ctypes.byref(jag(offsets=None))) == 0

    def call(d=None, j=None, q=fake(2), k=fake(3), v=fake(4), rp=fake(5), rt=fake(6), out=fake(7), ws=fake(8),
             ws_bytes=need):
        return L.hstu_attn_fwd(ctypes.byref(d or attn_desc()), ctypes.byref(j or jag()), q, k, v, rp, rt, out, ws,
                               ws_bytes, None)
    run_cases(L, call, [
        ("zero heads", dict(d=attn_desc(H=0)), INVALID),
        ("zero pos_max_len", dict(d=attn_desc(pos_max_len=0)), INVALID),
        ("zero buckets", dict(d=attn_desc(n_time_buckets=0)), UNSUPPORTED),
        ("129 buckets", dict(d=attn_desc(n_time_buckets=129)), UNSUPPORTED),
        ("inv_N not finite", dict(d=attn_desc(inv_N=float("nan"))), INVALID),
        ("F16 output", dict(d=attn_desc(o_dtype=F16)), UNSUPPORTED),
        ("unknown dtype", dict(d=attn_desc(dtype=7)), UNSUPPORTED),
        ("d = 32 on the tensor cores", dict(d=attn_desc(d_qk=32, d_v=32)), UNSUPPORTED),
        ("ld_q not a multiple of 8", dict(d=attn_desc(ld_q=1020)), UNSUPPORTED),
        ("ld_o below H d", dict(d=attn_desc(ld_o=64)), INVALID),
        ("F32 with d above 64", dict(d=attn_desc(dtype=F32, d_qk=65)), UNSUPPORTED),
        ("F32 inputs with BF16 output", dict(d=attn_desc(dtype=F32, o_dtype=BF16)), UNSUPPORTED),
        ("no workspace", dict(ws=None), INVALID),
        ("workspace one byte short", dict(ws_bytes=need - 1), WORKSPACE),
        ("no q", dict(q=None), INVALID),
        ("no rab_time", dict(rt=None), INVALID),
        ("out off 16 bytes", dict(out=fake(7) + 8), UNSUPPORTED),
        ("k off 16 bytes", dict(k=fake(3) + 2), UNSUPPORTED),
        ("no timestamps", dict(j=jag(timestamps=None)), INVALID),
        ("tile-pair rows beyond 32 bits", dict(j=jag(**HUGE_FWD)), UNSUPPORTED),
        ("the same on the CUDA-core path", dict(j=jag(**HUGE_FWD), d=attn_desc(dtype=F32, o_dtype=F32)), UNSUPPORTED),
    ])
    assert L.hstu_attn_workspace_size(ctypes.byref(attn_desc()), ctypes.byref(jag(**HUGE_FWD))) == 0
    assert L.hstu_attn_workspace_size(ctypes.byref(attn_desc()), ctypes.byref(jag(**HUGE_BWD))) > 0
    assert passes_host_checks(L, call, d=attn_desc(dtype=F32, d_qk=48, d_v=48))   # CUDA-core path: any d <= 64


def test_attn_fwd_noalloc(L):
    def call(d=None, j=None, q=fake(2), out=fake(7)):
        return L.hstu_attn_fwd_noalloc(ctypes.byref(d or attn_desc()), ctypes.byref(j or jag()), q, fake(3), fake(4),
                                       fake(5), fake(6), out, None)
    run_cases(L, call, [
        ("more work items than the fixed scratch holds", dict(j=jag(B=65536, T=300)), WORKSPACE),
        ("no q", dict(q=None), INVALID),
        ("out off 16 bytes", dict(out=fake(7) + 4), UNSUPPORTED),
        ("129 buckets", dict(d=attn_desc(n_time_buckets=129)), UNSUPPORTED),
        ("one sequence of 70,000 tiles", dict(j=jag(B=1, T=128 * 70000, max_len=1 << 30)), WORKSPACE),
    ])
    assert L.hstu_attn_fwd_noalloc_status(None, None) == INVALID


def test_attn_bwd(L):
    need = L.hstu_attn_bwd_workspace_size(ctypes.byref(attn_desc()), ctypes.byref(jag()))
    assert need > L.hstu_attn_workspace_size(ctypes.byref(attn_desc()), ctypes.byref(jag()))

    def call(d=None, j=None, q=fake(2), do=fake(5), dq=fake(8), drp=fake(11), drt=fake(12), ws=fake(13),
             ws_bytes=need):
        return L.hstu_attn_bwd(ctypes.byref(d or attn_desc()), ctypes.byref(j or jag()), q, fake(3), fake(4), do, fake(6),
                               fake(7), dq, fake(9), fake(10), drp, drt, ws, ws_bytes, None)
    run_cases(L, call, [
        ("F32 inputs (tensor cores only)", dict(d=attn_desc(dtype=F32, o_dtype=F32)), UNSUPPORTED),
        ("no workspace", dict(ws=None), INVALID),
        ("workspace one byte short", dict(ws_bytes=need - 1), WORKSPACE),
        ("no d rab_pos", dict(drp=None), INVALID),
        ("no d rab_time", dict(drt=None), INVALID),
        ("no q", dict(q=None), INVALID),
        ("no dout", dict(do=None), INVALID),
        ("dq off 16 bytes", dict(dq=fake(8) + 4), UNSUPPORTED),
        ("d = 32", dict(d=attn_desc(d_qk=32, d_v=32)), UNSUPPORTED),
        ("dX^T rows beyond 32 bits", dict(j=jag(**HUGE_BWD)), UNSUPPORTED),
    ])
    assert L.hstu_attn_bwd_workspace_size(ctypes.byref(attn_desc()), ctypes.byref(jag(**HUGE_BWD))) == 0
    # with one head the same batch fits the backward's bound
    assert L.hstu_attn_bwd_workspace_size(ctypes.byref(attn_desc(H=1, ld_q=64, ld_k=64, ld_v=64, ld_o=64)),
                                          ctypes.byref(jag(**HUGE_BWD))) > 0


def test_norm_gate_fwd(L):
    def call(T=300, D=256, odt=F32, udt=F16, gdt=F16, o=fake(2), ld_o=256, u=fake(3), ld_u=1024, gamma=fake(4),
             beta=fake(5), g=fake(6)):
        return L.hstu_norm_gate_fwd(T, D, odt, udt, gdt, o, ld_o, u, ld_u, gamma, beta, 1e-5, g, fake(7), fake(8),
                                    None)
    run_cases(L, call, [
        ("negative T", dict(T=-1), INVALID),
        ("BF16 o with F32 u", dict(odt=BF16, udt=F32, gdt=F32), UNSUPPORTED),
        ("F16 u with F32 g", dict(gdt=F32), UNSUPPORTED),
        ("D = 192", dict(D=192), UNSUPPORTED),
        ("no gamma", dict(gamma=None), INVALID),
        ("no g", dict(g=None), INVALID),
        ("ld_o below D", dict(ld_o=128), INVALID),
        ("ld_u not a multiple of 8", dict(ld_u=1028), UNSUPPORTED),
        ("gamma off 16 bytes", dict(gamma=fake(4) + 4), UNSUPPORTED),
        ("u off 16 bytes", dict(u=fake(3) + 2), UNSUPPORTED),
    ])
    assert attempt(L, call, T=0) == (OK, False)


def test_out_proj_fwd(L):
    need = L.hstu_out_proj_workspace_size(256, F16)
    assert need >= 256 + 256 * 256 * 2 and L.hstu_out_proj_workspace_size(256, BF16) == 256

    def call(D=256, dt=BF16, gdt=F16, g=fake(2), W2=fake(3), b2=fake(4), x=fake(5), xdt=BF16, y=fake(6), ydt=F32,
             y16=None, ws=fake(7), ws_bytes=need):
        return L.hstu_out_proj_fwd(300, D, dt, gdt, g, W2, b2, x, xdt, y, ydt, y16, ws, ws_bytes, None)
    run_cases(L, call, [
        ("F32 G with BF16 compute", dict(gdt=F32), UNSUPPORTED),
        ("workspace without the fp16 W2", dict(ws_bytes=256), WORKSPACE),
        ("F16 x", dict(xdt=F16), UNSUPPORTED),
        ("F32 compute with an fp16 copy of y", dict(dt=F32, gdt=F32, xdt=F32, y16=fake(8)), UNSUPPORTED),
        ("no W2", dict(W2=None), INVALID),
        ("no workspace", dict(ws=None), INVALID),
        ("b2 off 16 bytes", dict(b2=fake(4) + 4), UNSUPPORTED),
        ("y off 16 bytes", dict(y=fake(6) + 8), UNSUPPORTED),
    ])
    assert passes_host_checks(L, call, b2=None)


def test_linear_bf16(L):
    def call(M=296, N=256, K=320, A=fake(2), lda=320, a_mn=0, B=fake(3), ldb=320, b_mn=0, bias=fake(4), resid=fake(5),
             rdt=BF16, ld_r=256, out=fake(6), odt=F32, ld_o=256, acc=0, ws=fake(7), ws_bytes=256):
        return L.hstu_linear_bf16(M, N, K, A, lda, a_mn, B, ldb, b_mn, bias, resid, rdt, ld_r, out, odt, ld_o, acc, ws,
                                  ws_bytes, None)
    run_cases(L, call, [
        ("negative M", dict(M=-1), INVALID),
        ("no workspace", dict(ws=None), INVALID),
        ("workspace below 256 bytes", dict(ws_bytes=255), WORKSPACE),
        ("no A", dict(A=None), INVALID),
        ("N not a multiple of 32", dict(N=100), UNSUPPORTED),
        ("lda not a multiple of 8", dict(lda=324), UNSUPPORTED),
        ("lda below K (K-major A)", dict(lda=312), INVALID),
        ("lda below M (MN-major A)", dict(a_mn=1, lda=288), INVALID),
        ("ldb below N (MN-major B)", dict(b_mn=1, ldb=248), INVALID),
        ("ld_out below N", dict(ld_o=248), INVALID),
        ("ld_resid below N", dict(ld_r=248), INVALID),
        ("residual rows off 16 bytes", dict(ld_r=260), UNSUPPORTED),
        ("bias off 16 bytes", dict(bias=fake(4) + 4), UNSUPPORTED),
        ("resid off 16 bytes", dict(resid=fake(5) + 2), UNSUPPORTED),
        ("unknown residual dtype", dict(rdt=7), UNSUPPORTED),
        ("accumulate with a bias", dict(acc=1, resid=None), UNSUPPORTED),
        ("accumulate into BF16", dict(acc=1, bias=None, resid=None, odt=BF16), UNSUPPORTED),
        ("unknown output dtype", dict(odt=7), UNSUPPORTED),
    ])
    assert attempt(L, call, M=0) == (OK, False)
    assert passes_host_checks(L, call, a_mn=1, lda=296, b_mn=1, ldb=256)   # both MN-major, minimum strides
    assert passes_host_checks(L, call, acc=1, bias=None, resid=None, ld_r=0)   # no resid: ld_resid unread


def layer_desc(**kw):
    d = Hb.make_layer_desc(256, 4, 1.0 / 256, 256, BF16, BF16, BF16)
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def weights(**kw):
    names = ("W1", "b1", "W2", "b2", "gamma", "beta", "rab_pos", "rab_time")
    vals = {n: fake(20 + i) for i, n in enumerate(names)}
    vals.update(kw)
    return Hb.hstu_layer_weights_t(*[vals[n] for n in names])


def saved(**kw):
    names = ("uvqk", "z", "o", "g", "mu", "rstd", "attn_bias")
    vals = {n: fake(30 + i) for i, n in enumerate(names)}
    vals["attn_bias"] = None
    vals.update(kw)
    return Hb.hstu_layer_saved_t(*[vals[n] for n in names])


def test_layer_fwd(L):
    need = L.hstu_layer_workspace_size(ctypes.byref(layer_desc()), ctypes.byref(jag()))
    assert need >= L.hstu_attn_workspace_size(ctypes.byref(attn_desc()), ctypes.byref(jag()))

    def call(d=None, j=None, w=None, x=fake(2), y=fake(3), y16=None, sv=None, ws=fake(4), ws_bytes=need):
        return L.hstu_layer_fwd(ctypes.byref(d or layer_desc()), ctypes.byref(j or jag()), ctypes.byref(w or weights()), x,
                                None, y, y16, ctypes.byref(sv or saved()), ws, ws_bytes, None)
    run_cases(L, call, [
        ("D not divisible by H", dict(d=layer_desc(H=3)), INVALID),
        ("head width 32 on the tensor cores", dict(d=layer_desc(H=8)), UNSUPPORTED),
        ("129 buckets", dict(d=layer_desc(n_time_buckets=129)), UNSUPPORTED),
        ("F32 compute with an fp16 copy of y", dict(d=layer_desc(dtype=F32, x_dtype=F32, y_dtype=F32), y16=fake(5)),
         UNSUPPORTED),
        ("no workspace", dict(ws=None), INVALID),
        ("workspace one byte short", dict(ws_bytes=need - 1), WORKSPACE),
        ("no W1", dict(w=weights(W1=None)), INVALID),
        ("no rab_time", dict(w=weights(rab_time=None)), INVALID),
        ("no saved o", dict(sv=saved(o=None)), INVALID),
        ("no y", dict(y=None), INVALID),
        ("gamma off 16 bytes", dict(w=weights(gamma=fake(24) + 4)), UNSUPPORTED),
        ("beta off 16 bytes", dict(w=weights(beta=fake(25) + 4)), UNSUPPORTED),
        ("b1 off 16 bytes", dict(w=weights(b1=fake(21) + 4)), UNSUPPORTED),
        ("b2 off 16 bytes", dict(w=weights(b2=fake(23) + 4)), UNSUPPORTED),
        ("W2 off 16 bytes", dict(w=weights(W2=fake(22) + 2)), UNSUPPORTED),
        ("x off 16 bytes", dict(x=fake(2) + 2), UNSUPPORTED),
        ("bias cache off 256 bytes", dict(sv=saved(attn_bias=fake(36) + 128)), UNSUPPORTED),
        ("tile-pair rows beyond 32 bits", dict(j=jag(**HUGE_FWD)), UNSUPPORTED),
    ])
    assert L.hstu_layer_workspace_size(ctypes.byref(layer_desc()), ctypes.byref(jag(**HUGE_FWD))) == 0
    assert passes_host_checks(L, call, sv=saved(z=None))                   # z is optional in the forward
    # the CUDA-core path reads the biases one element at a time
    assert passes_host_checks(L, call, d=layer_desc(dtype=F32, x_dtype=F32, y_dtype=F32), w=weights(b1=fake(21) + 4))


def test_layer_bwd(L):
    need = L.hstu_layer_bwd_workspace_size(ctypes.byref(layer_desc()), ctypes.byref(jag()))
    assert need > 0

    def grads(**kw):
        names = ("dW1", "db1", "dW2", "db2", "dgamma", "dbeta", "drab_pos", "drab_time")
        vals = {n: fake(40 + i) for i, n in enumerate(names)}
        vals.update(kw)
        return Hb.hstu_layer_grads_t(*[vals[n] for n in names])

    def call(d=None, j=None, w=None, sv=None, gr=None, x=fake(2), dy=fake(3), dx=fake(4), ws=fake(5), ws_bytes=need):
        return L.hstu_layer_bwd(ctypes.byref(d or layer_desc()), ctypes.byref(j or jag()), ctypes.byref(w or weights()), x,
                                None, ctypes.byref(sv or saved()), dy, None, dx, None, ctypes.byref(gr or grads()), ws,
                                ws_bytes, None)
    run_cases(L, call, [
        ("F32 compute", dict(d=layer_desc(dtype=F32, x_dtype=F32, y_dtype=F32)), UNSUPPORTED),
        ("D = 128", dict(d=layer_desc(D=128, H=2)), UNSUPPORTED),
        ("F16 x", dict(d=layer_desc(x_dtype=F16)), UNSUPPORTED),
        ("no workspace", dict(ws=None), INVALID),
        ("workspace one byte short", dict(ws_bytes=need - 1), WORKSPACE),
        ("no d rab_pos", dict(gr=grads(drab_pos=None)), INVALID),
        ("no dy", dict(dy=None), INVALID),
        ("no saved z", dict(sv=saved(z=None)), INVALID),
        ("no W1", dict(w=weights(W1=None)), INVALID),
        ("no gamma", dict(w=weights(gamma=None)), INVALID),
        ("no rab_time", dict(w=weights(rab_time=None)), INVALID),
        ("gamma off 16 bytes", dict(w=weights(gamma=fake(24) + 4)), UNSUPPORTED),
        ("dW1 off 16 bytes", dict(gr=grads(dW1=fake(40) + 4)), UNSUPPORTED),
        ("dx off 16 bytes", dict(dx=fake(4) + 2), UNSUPPORTED),
        ("bias cache off 256 bytes", dict(sv=saved(attn_bias=fake(36) + 16)), UNSUPPORTED),
        ("dX^T rows beyond 32 bits", dict(j=jag(**HUGE_BWD)), UNSUPPORTED),
    ])
    assert L.hstu_layer_bwd_workspace_size(ctypes.byref(layer_desc()), ctypes.byref(jag(**HUGE_BWD))) == 0
    assert passes_host_checks(L, call, w=weights(b1=None, b2=None))   # the backward does not read the biases
    assert passes_host_checks(L, call, sv=saved(attn_bias=fake(36)))   # the optional bias cache


def test_layer_bias_cache_size(L):
    """48 KB per causal tile pair (a 32 KB half-bias tile and a 16 KB bucket tile) of the batch's
    pair bound, then the backward's work list; 0 for a refused descriptor or batch."""
    size = L.hstu_layer_bias_cache_size
    size.restype = ctypes.c_size_t
    # B = 2 sequences of at most 200 rows: 2 tiles each, so at most 3 causal pairs per sequence
    n = size(ctypes.byref(layer_desc()), ctypes.byref(jag()))
    assert n >= 6 * 48 * 1024 and n % 256 == 0
    assert size(None, ctypes.byref(jag())) == 0
    assert size(ctypes.byref(layer_desc()), ctypes.byref(jag(**HUGE_BWD))) == 0


def falcon_desc(**kw):
    d = Hb.hstu_falcon_desc_t(L=2, users=2, m=4, b_m=2, D=256, H=4, inv_N=1.0 / 256, pos_max_len=256,
                              n_time_buckets=128, ln_eps=1e-5)
    for k, v in kw.items():
        setattr(d, k, v)
    return d


def test_falcon_fwd(L):
    need = L.hstu_falcon_workspace_size(ctypes.byref(falcon_desc()), ctypes.byref(jag()))
    assert need > 0
    assert L.hstu_falcon_cache_size(ctypes.byref(falcon_desc()), ctypes.byref(jag())) == 2 * 300 * 2 * 256 * 2

    def call(d=None, j=None, layers=None, cand=fake(3), req=fake(4), out=fake(5), ws=fake(6), ws_bytes=need):
        arr = (Hb.hstu_layer_weights_t * 2)(*(layers or [weights(), weights()]))
        return L.hstu_falcon_fwd(ctypes.byref(d or falcon_desc()), arr, ctypes.byref(j or jag()), fake(2), fake(7), 0,
                                 None, cand, req, out, ws, ws_bytes, None)
    run_cases(L, call, [
        ("users differ from the prefix batch", dict(d=falcon_desc(users=3)), INVALID),
        ("zero micro-batch", dict(d=falcon_desc(b_m=0)), INVALID),
        ("zero layers", dict(d=falcon_desc(L=0)), INVALID),
        ("head width 32", dict(d=falcon_desc(H=8)), UNSUPPORTED),
        ("129 buckets", dict(d=falcon_desc(n_time_buckets=129)), UNSUPPORTED),
        ("inv_N not finite", dict(d=falcon_desc(inv_N=float("inf"))), INVALID),
        ("workspace one byte short", dict(ws_bytes=need - 1), WORKSPACE),
        ("no candidates", dict(cand=None), INVALID),
        ("no request times", dict(req=None), INVALID),
        ("out off 16 bytes", dict(out=fake(5) + 8), UNSUPPORTED),
        ("second layer without gamma", dict(layers=[weights(), weights(gamma=None)]), INVALID),
        ("second layer's gamma off 16 bytes", dict(layers=[weights(), weights(gamma=fake(24) + 4)]), UNSUPPORTED),
        ("second layer's b2 off 16 bytes", dict(layers=[weights(), weights(b2=fake(23) + 4)]), UNSUPPORTED),
        ("prefix tile-pair rows beyond 32 bits", dict(j=jag(**HUGE_FWD)), UNSUPPORTED),
    ])
    assert L.hstu_falcon_workspace_size(ctypes.byref(falcon_desc()), ctypes.byref(jag(**HUGE_FWD))) == 0
    assert attempt(L, call, d=falcon_desc(m=0)) == (OK, False)   # no candidates: nothing to do


def test_stochastic_length(L):
    def call(alpha=1.6, new_off=fake(2), ws=fake(3), ws_bytes=256, j=None):
        return L.hstu_stochastic_length_offsets(ctypes.byref(j or jag()), alpha, new_off, ws, ws_bytes, None)
    run_cases(L, call, [
        ("alpha above 2", dict(alpha=2.5), INVALID),
        ("negative alpha", dict(alpha=-0.1), INVALID),
        ("alpha NaN", dict(alpha=float("nan")), INVALID),
        ("no output offsets", dict(new_off=None), INVALID),
        ("no workspace", dict(ws=None), INVALID),
        ("workspace below 256 bytes", dict(ws_bytes=100), WORKSPACE),
        ("no offsets", dict(j=jag(offsets=None)), INVALID),
    ])


def test_stochastic_length_select(L):
    def call(keys=fake(2), new_off=fake(3), x=fake(4), xdt=BF16, D=256, kept=fake(5), x_out=fake(6), ws=fake(7),
             ws_bytes=256, j=None):
        return L.hstu_stochastic_length_select(ctypes.byref(j or jag()), keys, new_off, x, xdt, D, kept, x_out,
                                               fake(8), ws, ws_bytes, None)
    run_cases(L, call, [
        ("no keys", dict(keys=None), INVALID),
        ("no new offsets", dict(new_off=None), INVALID),
        ("no kept indices", dict(kept=None), INVALID),
        ("no workspace", dict(ws=None), INVALID),
        ("workspace below 256 bytes", dict(ws_bytes=8), WORKSPACE),
        ("rows out without rows in", dict(x=None), INVALID),
        ("zero width", dict(D=0), INVALID),
        ("unknown dtype", dict(xdt=7), UNSUPPORTED),
        ("rows not a multiple of 16 bytes", dict(D=100), UNSUPPORTED),
        ("x off 16 bytes", dict(x=fake(4) + 8), UNSUPPORTED),
        ("x_out off 16 bytes", dict(x_out=fake(6) + 2), UNSUPPORTED),
    ])
    assert passes_host_checks(L, call, x=None, x_out=None, D=0)     # indices only: x is not read
    assert attempt(L, call, j=jag(B=2, T=0)) == (OK, False)


def test_status_and_probe(L):
    st = ctypes.c_int32(0)
    assert L.hstu_sync_status(None, None, ctypes.byref(st)) == INVALID
    assert L.hstu_sync_status(fake(0), None, None) == INVALID
    assert L.hstu_debug_timeout_probe(None, 256, None) == INVALID
    assert L.hstu_debug_timeout_probe(fake(0), 255, None) == WORKSPACE
    for code, name in Hb.STATUS.items():
        assert L.hstu_status_string(code).decode() == name
    assert L.hstu_status_string(99).decode() == "HSTU_ERR_UNKNOWN"


def test_last_cuda_error_is_per_host_thread(L):
    """A CUDA failure on one host thread is not reported on another (the header's threading rule)."""
    import threading

    seen = {}

    def fresh_thread():
        seen["before"] = L.hstu_last_cuda_error()
        seen["marked"] = _mark_launch(L)

    _mark_encode(L)
    mine = L.hstu_last_cuda_error()
    t = threading.Thread(target=fresh_thread)
    t.start()
    t.join()
    assert seen["before"] == 0 and seen["marked"] != 0
    assert L.hstu_last_cuda_error() == mine != seen["marked"]


def test_profile_events(L):
    assert L.hstu_profile_events(7, fake(0), fake(1)) == INVALID        # no such kernel
    assert L.hstu_profile_events(-1, None, None) == INVALID
    assert L.hstu_profile_events(0, fake(0), None) == INVALID           # one event only
    assert L.hstu_profile_events(0, None, fake(1)) == INVALID
    for k in range(7):
        assert L.hstu_profile_events(k, None, None) == OK               # disabling is always fine


def rab_ext(**kw):
    e = Hb.hstu_rab_ext_t(per_head=1, n_types=3, token_type=fake(20), rab_type=fake(21))
    for k, v in kw.items():
        setattr(e, k, v)
    return e


def test_attn_fwd_ext(L):
    need = L.hstu_attn_ext_workspace_size(ctypes.byref(attn_desc()), ctypes.byref(jag()), ctypes.byref(rab_ext()))
    shared = L.hstu_attn_ext_workspace_size(ctypes.byref(attn_desc()), ctypes.byref(jag()),
                                            ctypes.byref(rab_ext(per_head=0)))
    assert need > shared == L.hstu_attn_workspace_size(ctypes.byref(attn_desc()), ctypes.byref(jag()))

    def call(d=None, j=None, e="default", q=fake(2), ws_bytes=need):
        ext = ctypes.byref(rab_ext()) if e == "default" else (None if e is None else ctypes.byref(e))
        return L.hstu_attn_fwd_ext(ctypes.byref(d or attn_desc()), ctypes.byref(j or jag()), ext, q, fake(3), fake(4),
                                   fake(5), fake(6), fake(7), fake(8), ws_bytes, None)
    run_cases(L, call, [
        ("no ext", dict(e=None), INVALID),
        ("per_head 2", dict(e=rab_ext(per_head=2)), INVALID),
        ("17 types", dict(e=rab_ext(n_types=17)), UNSUPPORTED),
        ("types without a type array", dict(e=rab_ext(token_type=None)), INVALID),
        ("types without a type table", dict(e=rab_ext(rab_type=None)), INVALID),
        ("workspace sized for shared tables", dict(ws_bytes=shared), WORKSPACE),
        ("fp32 descriptor", dict(d=attn_desc(dtype=F32, o_dtype=F32)), UNSUPPORTED),
        ("no q", dict(q=None), INVALID),
    ])
    assert passes_host_checks(L, call, e=rab_ext(n_types=0, token_type=None, rab_type=None))


def test_attn_bwd_ext(L):
    need = L.hstu_attn_bwd_ext_workspace_size(ctypes.byref(attn_desc()), ctypes.byref(jag()), ctypes.byref(rab_ext()))
    assert need > L.hstu_attn_bwd_workspace_size(ctypes.byref(attn_desc()), ctypes.byref(jag()))

    def call(e="default", drty=fake(14), ws_bytes=need):
        ext = ctypes.byref(rab_ext()) if e == "default" else (None if e is None else ctypes.byref(e))
        return L.hstu_attn_bwd_ext(ctypes.byref(attn_desc()), ctypes.byref(jag()), ext, fake(2), fake(3), fake(4),
                                   fake(5), fake(6), fake(7), fake(8), fake(9), fake(10), fake(11), fake(12), drty,
                                   fake(13), ws_bytes, None)
    run_cases(L, call, [
        ("no ext", dict(e=None), INVALID),
        ("types without d_rab_type", dict(drty=None), INVALID),
        ("small workspace", dict(ws_bytes=need - 1), WORKSPACE),
    ])
    assert passes_host_checks(L, call, e=rab_ext(n_types=0, token_type=None, rab_type=None), drty=None)


def test_falcon_append(L):
    old, app, new = jag(T=200), jag(T=100), jag(T=300)
    need = L.hstu_falcon_append_workspace_size(ctypes.byref(falcon_desc()), ctypes.byref(old), ctypes.byref(app),
                                               ctypes.byref(new))
    assert need > 0

    def call(d=None, o=None, a=None, n=None, layers=None, cache_old=fake(2), app_x=fake(3), cache_new=fake(4),
             out=fake(5), ws_bytes=need):
        arr = (Hb.hstu_layer_weights_t * 2)(*(layers or [weights(), weights()]))
        return L.hstu_falcon_append(ctypes.byref(d or falcon_desc()), arr, ctypes.byref(o or old), cache_old,
                                    ctypes.byref(a or app), app_x, ctypes.byref(n or new), cache_new, out, fake(6),
                                    ws_bytes, None)
    run_cases(L, call, [
        ("old and appended rows do not add up", dict(a=jag(T=99)), INVALID),
        ("appended batch with another user count", dict(a=jag(B=3, T=100)), INVALID),
        ("users differ from the combined batch", dict(d=falcon_desc(users=3)), INVALID),
        ("workspace one byte short", dict(ws_bytes=need - 1), WORKSPACE),
        ("no new cache", dict(cache_new=None), INVALID),
        ("no old cache", dict(cache_old=None), INVALID),
        ("no appended rows", dict(app_x=None), INVALID),
        ("new cache off 16 bytes", dict(cache_new=fake(4) + 2), UNSUPPORTED),
        ("second layer without W2", dict(layers=[weights(), weights(W2=None)]), INVALID),
        ("head width 32", dict(d=falcon_desc(H=8)), UNSUPPORTED),
    ])
