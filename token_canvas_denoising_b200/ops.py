"""Python wrappers of the single-operation entry points (include/dg_ops.h).

Marshalling only: torch tensors supply device memory and the stream; the
computation runs in libdgcanvas.so."""
import ctypes as C

import torch

from . import _lib as L


def _dt(t):
    if t.dtype == torch.float32:
        return L.DG_F32
    if t.dtype == torch.bfloat16:
        return L.DG_BF16
    raise TypeError(f"unsupported dtype {t.dtype}")


def _stream():
    return C.c_void_p(torch.cuda.current_stream().cuda_stream)


def _p(t):
    return C.c_void_p(t.data_ptr()) if t is not None else C.c_void_p(0)


def lmhead_entropy(hs, lm_head, inv_temp=None):
    """(entropy f32 [M], argmax int32 [M]) of softmax(hs @ lm_head.T * inv_temp)."""
    lib = L.load()
    M, d = hs.shape
    V = lm_head.shape[0]
    ent = torch.empty(M, dtype=torch.float32, device=hs.device)
    am = torch.empty(M, dtype=torch.int32, device=hs.device)
    st = lib.dg_lmhead_entropy(_dt(hs), _p(hs), _p(lm_head), _p(inv_temp), M, d, V, _p(ent), _p(am), _stream())
    L.check(st, "dg_lmhead_entropy")
    return ent, am


def lmhead_entropy_e4m3(hs, lm_codes, lm_scale, inv_temp=None):
    """The LM head with e4m3 weights: hs bf16 [M][d] (quantized per row inside),
    lm_codes uint8 [V][d] e4m3 codes, lm_scale f32 [V] row scales (powers of
    two). Returns (entropy f32 [M], argmax int32 [M])."""
    lib = L.load()
    M, d = hs.shape
    V = lm_codes.shape[0]
    ent = torch.empty(M, dtype=torch.float32, device=hs.device)
    am = torch.empty(M, dtype=torch.int32, device=hs.device)
    st = lib.dg_lmhead_entropy_e4m3(_p(hs), _p(lm_codes), _p(lm_scale), _p(inv_temp), M, d, V, _p(ent), _p(am),
                                    _stream())
    L.check(st, "dg_lmhead_entropy_e4m3")
    return ent, am


def lmhead_entropy_noalloc(hs, lm_head, inv_temp=None, ent=None, argmax=None):
    """Like lmhead_entropy, but the library makes no device allocation: its
    temporary partial results live in a fixed device array inside the library.
    Pass preallocated `ent` (f32 [M]) and `argmax` (int32 [M]) to allocate
    nothing on the Python side either."""
    lib = L.load()
    M, d = hs.shape
    V = lm_head.shape[0]
    if ent is None:
        ent = torch.empty(M, dtype=torch.float32, device=hs.device)
    if argmax is None:
        argmax = torch.empty(M, dtype=torch.int32, device=hs.device)
    st = lib.dg_lmhead_entropy_noalloc(_dt(hs), _p(hs), _p(lm_head), _p(inv_temp), M, d, V, _p(ent),
                                       _p(argmax), _stream())
    L.check(st, "dg_lmhead_entropy_noalloc")
    return ent, argmax


def attention(q, kc, vc, prefix_k, prefix_v, B, C_len, Hq, Hk, h):
    """Bidirectional GQA attention output [B*C, Hq*h] (see dg_ops.h)."""
    lib = L.load()
    o = torch.empty(B * C_len, Hq * h, dtype=q.dtype, device=q.device)
    plen = (C.c_int32 * B)(*[int(t.shape[0]) for t in prefix_k])
    pk = (C.c_void_p * B)(*[t.data_ptr() if t.numel() else None for t in prefix_k])
    pv = (C.c_void_p * B)(*[t.data_ptr() if t.numel() else None for t in prefix_v])
    st = lib.dg_attention(_dt(q), _p(q), _p(kc), _p(vc), B, C_len, Hq, Hk, h, C.cast(plen, C.c_void_p),
                          C.cast(pk, C.c_void_p), C.cast(pv, C.c_void_p), _p(o), _stream())
    L.check(st, "dg_attention")
    return o


def linear(a, w, residual=None):
    """a @ w.T (+ residual), f32 accumulate, output in a's dtype."""
    lib = L.load()
    M, K = a.shape
    N = w.shape[0]
    out = torch.empty(M, N, dtype=a.dtype, device=a.device)
    st = lib.dg_linear(_dt(a), _p(a), _p(w), _p(residual), _p(out), M, N, K, _stream())
    L.check(st, "dg_linear")
    return out
