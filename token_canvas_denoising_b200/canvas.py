"""Python binding of libdgcanvas: a thin object over the C ABI.

PyTorch provides device memory and streams only; the denoise path runs in the
CUDA library (see include/dg_canvas.h for what each call computes).
"""
import ctypes as C

import numpy as np
import torch

from . import _lib as L

_DT = {"f32": L.DG_F32, "bf16": L.DG_BF16}


def _ptr(t):
    return C.c_void_p(t.data_ptr()) if t is not None else C.c_void_p(0)


def to_device(arr, dtype, device):
    """numpy storage array (uint16 bf16 bits or float32) -> contiguous torch tensor."""
    t = torch.from_numpy(np.ascontiguousarray(arr))
    if arr.dtype == np.uint16:  # bf16 bit patterns (uint8 e4m3 codes stay bytes)
        t = t.view(torch.bfloat16)
    return t.to(device, non_blocking=False).contiguous()


def schedule(max_steps=48, stop_entropy=0.05, adaptive_stop=True):
    return L.dg_schedule(int(max_steps), float(stop_entropy), 1 if adaptive_stop else 0, L.DG_SCHED_CEIL)


class DenoiseCanvas:
    """A decode context for B canvases of C positions.

    weights: dict of device tensors in the storage dtype: embed, wq, wk, wv, wo,
    lm_head (+ w_router, w_gate, w_up, w_down for MoE). prefix_k / prefix_v:
    lists of B device tensors [S_b, Hk, h]. inv_temp: device f32 [B*C] or None.
    """

    def __init__(self, weights, *, d_model, n_q_heads, n_kv_heads, head_dim, vocab, dtype,
                 canvas_len, prefix_k, prefix_v, seeds, inv_temp=None, n_experts=0, top_k=0,
                 moe_inter=0, n_shared=0, n_layers=0, stream=None):
        self._lib = L.load()
        self.B = len(seeds)
        self.C = int(canvas_len)
        self.M = self.B * self.C
        self.dtype = dtype
        self._keep = [weights, prefix_k, prefix_v, inv_temp]  # keep caller memory alive
        m = L.dg_model_desc()
        m.d_model, m.n_q_heads, m.n_kv_heads, m.head_dim, m.vocab = d_model, n_q_heads, n_kv_heads, head_dim, vocab
        m.dtype = _DT[dtype]
        for k in ("embed", "wq", "wk", "wv", "wo", "lm_head"):
            setattr(m, k, weights[k].data_ptr())
        m.n_experts, m.top_k, m.moe_inter, m.n_shared = n_experts, top_k, moe_inter, n_shared
        m.n_layers = n_layers
        self.L = max(1, n_layers)
        if "lm_head_scale" in weights:  # e4m3 LM head
            m.lm_head_format = L.DG_LM_E4M3
            m.lm_head_scale = weights["lm_head_scale"].data_ptr()
        if n_experts:
            for k in ("w_router", "w_gate", "w_up", "w_down"):
                setattr(m, k, weights[k].data_ptr())
            if "w_gate_scale" in weights:  # e4m3 experts
                m.expert_format = L.DG_LM_E4M3
                for k in ("w_gate_scale", "w_up_scale", "w_down_scale"):
                    setattr(m, k, weights[k].data_ptr())
        self._model = m
        plen = (C.c_int32 * self.B)(*[self._plen(t) for t in prefix_k])
        pk = (C.c_void_p * self.B)(*[t.data_ptr() if t is not None and t.numel() else None for t in prefix_k])
        pv = (C.c_void_p * self.B)(*[t.data_ptr() if t is not None and t.numel() else None for t in prefix_v])
        sd = (C.c_uint64 * self.B)(*[int(s) for s in seeds])
        self.stream = stream if stream is not None else torch.cuda.current_stream()
        ctx = C.c_void_p()
        st = self._lib.dg_canvas_init(C.byref(ctx), C.byref(m), self.B, self.C, C.cast(plen, C.c_void_p),
                                      C.cast(pk, C.c_void_p), C.cast(pv, C.c_void_p), _ptr(inv_temp),
                                      C.cast(sd, C.c_void_p), C.c_void_p(self.stream.cuda_stream))
        L.check(st, "dg_canvas_init")
        self._ctx = ctx

    def _plen(self, t):
        """Prompt length of a cache tensor ([S][Hk][h], or [L][S][Hk][h] with L layers)."""
        if t is None:
            return 0
        return int(t.shape[1]) if self._model.n_layers > 0 and t.dim() == 4 else int(t.shape[0])

    # ------------------------------------------------------------------
    def step(self, sched, debug=False):
        """One denoise step; with debug=True returns the per-step outputs."""
        out = None
        dbg = None
        if debug:
            dev = torch.device("cuda", torch.cuda.current_device())
            sdt = torch.float32 if self.dtype == "f32" else torch.bfloat16
            qd = self._model.n_q_heads * self._model.head_dim
            kd = self._model.n_kv_heads * self._model.head_dim
            out = {
                "ent": torch.empty(self.M, dtype=torch.float32, device=dev),
                "argmax": torch.empty(self.M, dtype=torch.int32, device=dev),
                "freeze_mask": torch.empty(self.M, dtype=torch.uint8, device=dev),
                "attn_out": torch.empty(self.M, self._model.n_q_heads * self._model.head_dim, dtype=sdt, device=dev),
                "hidden": torch.empty(self.M, self._model.d_model, dtype=sdt, device=dev),
                "hidden_attn": torch.empty(self.M, self._model.d_model, dtype=sdt, device=dev),
                "q": torch.empty(self.M, qd, dtype=sdt, device=dev),
                "k_canvas": torch.empty(self.M, kd, dtype=sdt, device=dev),
                "v_canvas": torch.empty(self.M, kd, dtype=sdt, device=dev),
                "layer_out": torch.empty(self.L, self.M, self._model.d_model, dtype=sdt, device=dev),
            }
            dbg = L.dg_step_out(*[_ptr(out[k]) for k in ("ent", "argmax", "freeze_mask", "attn_out", "hidden",
                                                          "hidden_attn", "q", "k_canvas", "v_canvas", "layer_out")])
        st = self._lib.dg_denoise_step(self._ctx, C.byref(sched), C.byref(dbg) if dbg is not None else None)
        L.check(st, "dg_denoise_step")
        return out

    def decode(self, sched, tokens_out=None):
        """Denoise to completion. tokens_out: torch tensor (device or host int32
        [B*C]) or None for a fresh host tensor. Returns (tokens, steps)."""
        if tokens_out is None:
            tokens_out = torch.empty(self.M, dtype=torch.int32)
        steps = (C.c_int32 * self.B)()
        st = self._lib.dg_decode_block(self._ctx, C.byref(sched), _ptr(tokens_out), C.cast(steps, C.c_void_p))
        L.check(st, "dg_decode_block")
        return tokens_out, list(steps)

    def get_state(self):
        s = {"tokens": np.zeros(self.M, np.int32), "frozen": np.zeros(self.M, np.uint8),
             "step": np.zeros(self.B, np.int32), "seed": np.zeros(self.B, np.uint64),
             "done": np.zeros(self.B, np.uint8)}
        hs = L.dg_state(*[s[k].ctypes.data for k in ("tokens", "frozen", "step", "seed", "done")])
        L.check(self._lib.dg_canvas_get_state(self._ctx, C.byref(hs)), "dg_canvas_get_state")
        return s

    def set_state(self, s):
        arrs = {"tokens": np.ascontiguousarray(s["tokens"], np.int32).reshape(-1),
                "frozen": np.ascontiguousarray(s["frozen"], np.uint8).reshape(-1),
                "step": np.ascontiguousarray(s["step"], np.int32).reshape(-1),
                "seed": np.ascontiguousarray(s["seed"], np.uint64).reshape(-1),
                "done": np.ascontiguousarray(s["done"], np.uint8).reshape(-1)}
        hs = L.dg_state(*[arrs[k].ctypes.data for k in ("tokens", "frozen", "step", "seed", "done")])
        L.check(self._lib.dg_canvas_set_state(self._ctx, C.byref(hs)), "dg_canvas_set_state")

    def reset(self, seeds=None, fixed_mask=None, fixed_tokens=None):
        """Redraw every canvas at step 0 (device side, asynchronous). With
        fixed_mask / fixed_tokens ([B][C] or [B*C] arrays), the given positions
        take the given tokens and start frozen (synchronous)."""
        arr = None
        if seeds is not None:
            arr = (C.c_uint64 * self.B)(*[int(x) for x in seeds])
        seeds_p = C.cast(arr, C.c_void_p) if arr is not None else None
        if fixed_mask is None:
            st = self._lib.dg_canvas_reset(self._ctx, seeds_p)
            L.check(st, "dg_canvas_reset")
            return
        import numpy as np
        mask = np.ascontiguousarray(np.asarray(fixed_mask).reshape(-1) != 0, dtype=np.uint8)
        toks = np.ascontiguousarray(np.asarray(fixed_tokens).reshape(-1), dtype=np.int32)
        if mask.size != self.M or toks.size != self.M:
            raise ValueError(f"fixed_mask and fixed_tokens need {self.M} entries")
        st = self._lib.dg_canvas_reset_fixed(self._ctx, seeds_p, mask.ctypes.data_as(C.c_void_p),
                                             toks.ctypes.data_as(C.c_void_p))
        L.check(st, "dg_canvas_reset_fixed")

    def block_kv(self):
        """K and V of the current canvas tokens (the committed block), device
        tensors [B*C, Hk*h] in the storage dtype, canvas-major."""
        sdt = torch.float32 if self.dtype == "f32" else torch.bfloat16
        kd = self._model.n_kv_heads * self._model.head_dim
        dev = torch.device("cuda", torch.cuda.current_device())
        k = torch.empty(self.M, kd, dtype=sdt, device=dev)
        v = torch.empty(self.M, kd, dtype=sdt, device=dev)
        st = self._lib.dg_canvas_block_kv(self._ctx, _ptr(k), _ptr(v))
        L.check(st, "dg_canvas_block_kv")
        return k, v

    def set_prefix(self, prefix_k, prefix_v):
        """Attend to new prompt caches from the next step on: lists of B device
        tensors [S_b, Hk, h] (kept alive by this object)."""
        plen = (C.c_int32 * self.B)(*[self._plen(t) for t in prefix_k])
        pk = (C.c_void_p * self.B)(*[t.data_ptr() if t is not None and t.numel() else None for t in prefix_k])
        pv = (C.c_void_p * self.B)(*[t.data_ptr() if t is not None and t.numel() else None for t in prefix_v])
        st = self._lib.dg_canvas_set_prefix(self._ctx, C.cast(plen, C.c_void_p), C.cast(pk, C.c_void_p),
                                            C.cast(pv, C.c_void_p))
        L.check(st, "dg_canvas_set_prefix")
        self._keep[1], self._keep[2] = prefix_k, prefix_v

    def set_timing_events(self, starts, stops, kernel="lmhead"):
        """Record torch.cuda.Event pairs around one kernel of graph steps
        (pair i on step i mod n): kernel "lmhead" or "attention"; or one pair
        around the device-side loop of decode(): kernel "decode". Pass empty
        lists to turn off."""
        k = {"lmhead": L.DG_KERNEL_LMHEAD, "attention": L.DG_KERNEL_ATTENTION, "decode": L.DG_KERNEL_DECODE}[kernel]
        n = len(starts)
        a = (C.c_void_p * max(n, 1))(*[e.cuda_event for e in starts])
        b = (C.c_void_p * max(n, 1))(*[e.cuda_event for e in stops])
        st = self._lib.dg_canvas_set_kernel_timing(self._ctx, k, n, C.cast(a, C.c_void_p), C.cast(b, C.c_void_p))
        L.check(st, "dg_canvas_set_kernel_timing")

    def loop_steps(self):
        """Steps run by the device-side loop of the most recent decode()."""
        n = C.c_int32(0)
        L.check(self._lib.dg_canvas_loop_steps(self._ctx, C.byref(n)), "dg_canvas_loop_steps")
        return int(n.value)

    def sync(self):
        L.check(self._lib.dg_canvas_sync(self._ctx), "dg_canvas_sync")

    @property
    def launches_per_step(self):
        return int(self._lib.dg_launches_per_step(self._ctx))

    def close(self):
        if getattr(self, "_ctx", None):
            self._lib.dg_canvas_destroy(self._ctx)
            self._ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def from_workload(wl, device=None, stream=None):
    """Upload a seeded Workload (token_canvas_denoising_b200.inputs) and create a
    DenoiseCanvas over it. Returns (canvas, device tensors)."""
    c = wl.cfg
    device = device or torch.device("cuda", torch.cuda.current_device())
    w = {k: to_device(v, c.dtype, device) for k, v in wl.weights.items()}
    pk = [to_device(x, c.dtype, device) for x in wl.prefix_k]
    pv = [to_device(x, c.dtype, device) for x in wl.prefix_v]
    invT = None if c.inv_temp == "one" else torch.from_numpy(wl.inv_temp).to(device)
    cv = DenoiseCanvas(w, d_model=c.d, n_q_heads=c.Hq, n_kv_heads=c.Hk, head_dim=c.h, vocab=c.V,
                       dtype=c.dtype, canvas_len=c.C, prefix_k=pk, prefix_v=pv, seeds=list(wl.seeds),
                       inv_temp=invT, n_experts=c.n_experts, top_k=c.top_k, moe_inter=c.moe_inter,
                       n_shared=c.n_shared, n_layers=c.n_layers, stream=stream)
    return cv, {"weights": w, "prefix_k": pk, "prefix_v": pv, "inv_temp": invT}
