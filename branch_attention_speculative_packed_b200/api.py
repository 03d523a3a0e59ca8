"""PyTorch-facing wrappers of the C ABI.

PyTorch provides device memory (outputs, workspace) and the current CUDA
stream; the computation itself runs in libba_b200.so.  Tensor layouts are
those of include/ba.h: q [S,Hq,d], k/v [S,Hkv,d], qb [Nb,B,Hq,d],
kb/vb [Nb,B,Hkv,d], bf16, contiguous; LSE fp32 [Hq, S+Nb*B].
"""
from __future__ import annotations

import ctypes

import torch

from . import _abi
from ._abi import BA_WS_BWD, BA_WS_FWD, BaProblem, check


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


class BranchAttention:
    """One packing (documents + anchors) and the shape of its heads.

    cu_seqlens: int32 [ndoc+1]; anchors: int32 [Nb] ascending; B: branch depth
    (chain) or block size (block); mode: 0 chain (EAGLE-3 training-time test),
    1 block (DFlash-style), 2 bitmask (``branch_mask``: [Nb, B] 64-bit words,
    row (b, t) sees branch key u iff bit u of branch_mask[b, t]); R: virtual
    zigzag ranks; scale: softmax scale (None: 1/sqrt(d)); window: main-prefix
    window W (0: none); cp_rank: compute only virtual rank cp_rank's rows (its
    share under context parallelism; see include/ba.h)."""

    def __init__(self, cu_seqlens, anchors, *, Hq, Hkv, d, B, mode, R=1, scale=None,
                 device="cuda", window=0, branch_mask=None, cp_rank=None):
        self.cu_h = torch.as_tensor(cu_seqlens, dtype=torch.int32).cpu().contiguous()
        self.anc_h = torch.as_tensor(anchors, dtype=torch.int32).cpu().contiguous()
        self.device = torch.device(device)
        if self.device.type == "cuda":
            self.cu_d = self.cu_h.to(self.device)
            self.anc_d = self.anc_h.to(self.device) if self.anc_h.numel() else \
                torch.zeros(4, dtype=torch.int32, device=self.device)
        else:  # host-only use (planning statistics, workspace sizes)
            self.cu_d = self.cu_h
            self.anc_d = self.anc_h if self.anc_h.numel() else torch.zeros(4, dtype=torch.int32)
        self.S = int(self.cu_h[-1])
        self.ndoc = int(self.cu_h.numel() - 1)
        self.Nb = int(self.anc_h.numel())
        self.Hq, self.Hkv, self.d, self.B, self.mode, self.R = Hq, Hkv, d, B, mode, R
        self.scale = -1.0 if scale is None else float(scale)
        self.window = int(window)
        # None: every row; r: only the rows the zigzag split gives virtual rank r
        self.cp_rank = None if cp_rank is None else int(cp_rank)
        self.bm_h = self.bm_d = None
        if branch_mask is not None:
            bm = torch.as_tensor(branch_mask)
            if bm.dtype != torch.int64:  # uint64 words from numpy: keep the bits
                bm = torch.from_numpy(__import__("numpy").asarray(branch_mask).astype("uint64").view("int64"))
            self.bm_h = bm.reshape(-1).cpu().contiguous()
            self.bm_d = self.bm_h.to(self.device) if self.device.type == "cuda" else self.bm_h
        self._ws = {}

    @property
    def rows(self) -> int:
        return self.S + self.Nb * self.B

    def _problem(self, q=None, k=None, v=None, qb=None, kb=None, vb=None, ws=None) -> BaProblem:
        p = BaProblem()
        p.S, p.ndoc, p.Hq, p.Hkv, p.d = self.S, self.ndoc, self.Hq, self.Hkv, self.d
        p.Nb, p.B, p.mode, p.R, p.scale = self.Nb, self.B, self.mode, self.R, self.scale
        p.cu_seqlens_h = self.cu_h.data_ptr()
        p.cu_seqlens_d = self.cu_d.data_ptr()
        p.anchors_h = self.anc_h.data_ptr() if self.Nb else None
        p.anchors_d = self.anc_d.data_ptr() if self.Nb else None
        p.window = self.window
        if self.cp_rank is not None:
            p.cp_select, p.cp_rank = 1, self.cp_rank
        if self.bm_h is not None:
            p.branch_mask_h = self.bm_h.data_ptr()
            p.branch_mask_d = self.bm_d.data_ptr()
        for name, t in (("q", q), ("k", k), ("v", v), ("qb", qb), ("kb", kb), ("vb", vb)):
            if t is not None:
                if not t.is_contiguous() or t.dtype != torch.bfloat16:
                    raise ValueError(f"{name} must be a contiguous bf16 tensor")
                setattr(p, name, t.data_ptr() if t.numel() else None)
        if ws is not None:
            p.workspace = ws.data_ptr()
            p.workspace_bytes = ws.numel()
        return p

    def workspace_size(self, which: int) -> int:
        n = _abi.lib().ba_workspace_size(ctypes.byref(self._problem()), which)
        if n == 0:
            raise ValueError("invalid branch-attention problem")
        return int(n)

    def workspace(self, which: int) -> torch.Tensor:
        n = self.workspace_size(which)
        ws = self._ws.get(which)
        if ws is None or ws.numel() < n:
            ws = torch.empty(n + 256, dtype=torch.uint8, device=self.device)
            self._ws[which] = ws
        return ws

    def plan_stats(self):
        a, b, c = ctypes.c_int64(), ctypes.c_int64(), ctypes.c_int64()
        check(_abi.lib().ba_plan_stats(ctypes.byref(self._problem()), ctypes.byref(a),
                                       ctypes.byref(b), ctypes.byref(c)), "ba_plan_stats")
        return {"row_tiles": a.value, "tile_pairs": b.value, "visible_pairs": c.value}

    def prepare(self) -> float:
        """Build (or find) this problem's host plan in the library's cache;
        returns the host milliseconds building it took (ba_plan_prepare)."""
        ms = ctypes.c_double()
        check(_abi.lib().ba_plan_prepare(ctypes.byref(self._problem()), ctypes.byref(ms)),
              "ba_plan_prepare")
        return ms.value

    def rank_work(self):
        """(row tile, main key tile) pairs owned by each of the R virtual ranks."""
        buf = (ctypes.c_int64 * self.R)()
        n = _abi.lib().ba_plan_rank_work(ctypes.byref(self._problem()), buf, self.R)
        if n < 0:
            check(n, "ba_plan_rank_work")
        return list(buf)

    def fwd_pairs(self):
        """Forward work items: (tile, tile or -1) pairs in claim order."""
        n = _abi.lib().ba_plan_fwd_pairs(ctypes.byref(self._problem()), None, 0)
        if n < 0:
            check(n, "ba_plan_fwd_pairs")
        buf = (ctypes.c_int32 * (2 * max(n, 1)))()
        _abi.lib().ba_plan_fwd_pairs(ctypes.byref(self._problem()), buf, n)
        return [(buf[2 * i], buf[2 * i + 1]) for i in range(n)]

    # ------------------------------------------------------------------ forward
    def fused_fwd(self, q, k, v, qb, kb, vb, out=None, stream=None):
        """Steps a2+a3+a4: returns (o bf16 [S,Hq,d], ob bf16 [Nb,B,Hq,d], lse fp32 [Hq,rows])."""
        dev = q.device
        if out is None:
            o = torch.empty_like(q)
            ob = torch.empty(self.Nb, self.B, self.Hq, self.d, dtype=torch.bfloat16, device=dev)
            lse = torch.empty(self.Hq, self.rows, dtype=torch.float32, device=dev)
        else:
            o, ob, lse = out
        ws = self.workspace(BA_WS_FWD)
        p = self._problem(q, k, v, qb, kb, vb, ws)
        check(_abi.lib().ba_fused_fwd(ctypes.byref(p), _ptr(o), _ptr(ob) if self.Nb else None,
                                      _ptr(lse), _stream(stream)), "ba_fused_fwd")
        return o, ob, lse

    def fused_fwd_noalloc(self, q, k, v, qb, kb, vb, out, stream=None):
        """ba_fused_fwd for callers that cannot allocate: scratch comes from the
        library's static device array (no workspace); outputs must be given."""
        o, ob, lse = out
        p = self._problem(q, k, v, qb, kb, vb)
        check(_abi.lib().ba_fused_fwd_noalloc(ctypes.byref(p), _ptr(o), _ptr(ob) if self.Nb else None,
                                              _ptr(lse), _stream(stream)), "ba_fused_fwd_noalloc")
        return o, ob, lse

    def main_fwd(self, q, k, v, qb, kb, vb, stream=None):
        """Step a2: (o_part fp32 [rows,Hq,d], lse_part fp32 [Hq,rows])."""
        dev = q.device
        o = torch.empty(self.rows, self.Hq, self.d, dtype=torch.float32, device=dev)
        lse = torch.empty(self.Hq, self.rows, dtype=torch.float32, device=dev)
        ws = self.workspace(BA_WS_FWD)
        p = self._problem(q, k, v, qb, kb, vb, ws)
        check(_abi.lib().ba_main_fwd(ctypes.byref(p), _ptr(o), _ptr(lse), _stream(stream)),
              "ba_main_fwd")
        return o, lse

    def main_fwd_ring(self, q, k, v, qb, kb, vb, stream=None):
        """Step a2 by ring steps: partial k of every row over the visible main
        keys of virtual rank k's zigzag chunks.  Returns (o_parts fp32
        [R,rows,Hq,d], lse_parts fp32 [R,Hq,rows])."""
        dev = q.device
        o = torch.empty(self.R, self.rows, self.Hq, self.d, dtype=torch.float32, device=dev)
        lse = torch.empty(self.R, self.Hq, self.rows, dtype=torch.float32, device=dev)
        ws = self.workspace(BA_WS_FWD)
        p = self._problem(q, k, v, qb, kb, vb, ws)
        check(_abi.lib().ba_main_fwd_ring(ctypes.byref(p), _ptr(o), _ptr(lse), _stream(stream)),
              "ba_main_fwd_ring")
        return o, lse

    def branch_fwd(self, q, k, v, qb, kb, vb, stream=None):
        """Step a3: (o_part fp32 [Nb*B,Hq,d], lse_part fp32 [Hq,Nb*B])."""
        dev = q.device
        n = self.Nb * self.B
        o = torch.empty(n, self.Hq, self.d, dtype=torch.float32, device=dev)
        lse = torch.empty(self.Hq, n, dtype=torch.float32, device=dev)
        p = self._problem(q, k, v, qb, kb, vb)
        check(_abi.lib().ba_branch_fwd(ctypes.byref(p), _ptr(o), _ptr(lse), _stream(stream)),
              "ba_branch_fwd")
        return o, lse

    # ------------------------------------------------------------------ backward
    def bwd(self, q, k, v, qb, kb, vb, o, ob, lse, do, dob, out=None, stream=None):
        """Gradients of sum(O*dO): (dq, dk, dv, dqb, dkb, dvb), bf16, input layouts."""
        if out is None:
            out = (torch.empty_like(q), torch.empty_like(k), torch.empty_like(v),
                   torch.empty_like(qb), torch.empty_like(kb), torch.empty_like(vb))
        dq, dk, dv, dqb, dkb, dvb = out
        ws = self.workspace(BA_WS_BWD)
        p = self._problem(q, k, v, qb, kb, vb, ws)
        nb = self.Nb > 0
        check(_abi.lib().ba_bwd(ctypes.byref(p), _ptr(o), _ptr(ob) if nb else None, _ptr(lse),
                                _ptr(do), _ptr(dob) if nb else None, _ptr(dq), _ptr(dk), _ptr(dv),
                                _ptr(dqb) if nb else None, _ptr(dkb) if nb else None,
                                _ptr(dvb) if nb else None, _stream(stream)), "ba_bwd")
        return dq, dk, dv, dqb, dkb, dvb


def lse_merge(o_parts, lse_parts, out=None, stream=None):
    """Step a4, Eq. 2 over k partials: o_parts fp32 [rows,H,d] each, lse_parts
    fp32 2-D [H, >=rows] views (head stride = stride(0)).  Returns (o bf16, lse fp32 [H,rows])."""
    k = len(o_parts)
    rows, H, d = o_parts[0].shape
    if out is None:
        o = torch.empty(rows, H, d, dtype=torch.bfloat16, device=o_parts[0].device)
        lse = torch.empty(H, rows, dtype=torch.float32, device=o_parts[0].device)
    else:
        o, lse = out
    VP = ctypes.c_void_p * k
    I64 = ctypes.c_int64 * k
    for t in lse_parts:
        if t.stride(1) != 1:
            raise ValueError("LSE parts must have unit stride along rows")
    check(_abi.lib().ba_lse_merge(k, rows, H, d, VP(*[t.data_ptr() for t in o_parts]),
                                  VP(*[t.data_ptr() for t in lse_parts]),
                                  I64(*[t.stride(0) for t in lse_parts]), _ptr(o), _ptr(lse),
                                  lse.stride(0), _stream(stream)), "ba_lse_merge")
    return o, lse


def sync_status(stream=None) -> None:
    """Synchronise and raise BAError if a device-side bounded wait expired."""
    check(_abi.lib().ba_sync_status(_stream(stream)), "ba_sync_status")
