"""Python binding of libsageb200.so -- argument marshalling only.

Every step of the method runs in the library's CUDA kernels; this module only
checks shapes/dtypes, hands device pointers and the current CUDA stream to
the C ABI, and turns error codes into exceptions.  PyTorch provides device
memory and streams.
"""
from __future__ import annotations

import ctypes
import dataclasses
import math
from typing import Optional, Sequence

import torch

from . import _lib

F16, BF16, F32 = 0, 1, 2
PV_MODES = {"fp16": 0, "fp8": 1}
BLOCK = 128

STATUS = {
    0: "SAGE_OK", 1: "SAGE_ERR_INVALID_ARG", 2: "SAGE_ERR_UNSUPPORTED", 3: "SAGE_ERR_WORKSPACE",
    4: "SAGE_ERR_CUDA", 5: "SAGE_ERR_TIMEOUT", 6: "SAGE_ERR_BAD_SEQLENS", 7: "SAGE_ERR_RANGE",
}


class SageError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        name = STATUS.get(code, f"status {code}")
        detail = ""
        if code == 4:
            detail = _lib.load().sage_last_cuda_error().decode(errors="replace")
        super().__init__(f"{what}: {name}" + (f" ({detail})" if detail else ""))


def _check(code: int, what: str) -> None:
    if code != 0:
        raise SageError(code, what)


def _dtype_code(t: torch.dtype, allow_f32: bool = False) -> int:
    if t == torch.float16:
        return F16
    if t == torch.bfloat16:
        return BF16
    if allow_f32 and t == torch.float32:
        return F32
    raise ValueError(f"unsupported dtype {t}")


def _pv(pv_mode: str) -> int:
    if pv_mode not in PV_MODES:
        raise ValueError(f"pv_mode must be one of {sorted(PV_MODES)}")
    return PV_MODES[pv_mode]


def _stream(dev: torch.device) -> int:
    return torch.cuda.current_stream(dev).cuda_stream


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _need_cuda_contig(*ts: torch.Tensor) -> None:
    for t in ts:
        if not t.is_cuda:
            raise ValueError("tensors must be on a CUDA device")
        if not t.is_contiguous():
            raise ValueError("tensors must be contiguous")


class Workspace:
    """A caller-owned device workspace (torch uint8 buffer) with its status word."""

    def __init__(self, nbytes: int, device: torch.device | str | int = "cuda"):
        self.device = torch.device(device)
        self.buf = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=self.device)
        _check(_lib.load().sage_workspace_init(self.ptr, self.nbytes, _stream(self.device)),
               "sage_workspace_init")

    @property
    def ptr(self) -> int:
        return self.buf.data_ptr()

    @property
    def nbytes(self) -> int:
        return self.buf.numel()

    def ensure(self, nbytes: int) -> "Workspace":
        if nbytes > self.nbytes:
            self.__init__(nbytes, self.device)
        return self

    def sync_status(self) -> None:
        """Synchronise the current stream and raise on any device-side error."""
        _check(_lib.load().sage_sync_status(self.ptr, _stream(self.device)), "device status")


_default_ws: dict = {}


def _workspace(dev: torch.device, nbytes: int, ws: Optional[Workspace]) -> Workspace:
    if ws is not None:
        return ws.ensure(nbytes)
    key = (dev.index if dev.index is not None else torch.cuda.current_device())
    w = _default_ws.get(key)
    if w is None:
        w = _default_ws[key] = Workspace(nbytes, dev)
    return w.ensure(nbytes)


def workspace_bytes(B: int, H: int, N: int, D: int, pv_mode: str = "fp16") -> int:
    return int(_lib.load().sage_workspace_bytes(B, H, N, D, _pv(pv_mode)))


def workspace_bytes_gqa(B: int, H: int, Hkv: int, N: int, D: int, pv_mode: str = "fp16") -> int:
    """Workspace of attn_fwd with [B, H, N, D] queries over [B, Hkv, N, D] keys/values."""
    return int(_lib.load().sage_workspace_bytes_gqa(B, H, Hkv, N, D, _pv(pv_mode)))


def workspace_bytes_varlen(total_tokens: int, batch: int, H: int, D: int,
                           pv_mode: str = "fp16") -> int:
    return int(_lib.load().sage_workspace_bytes_varlen(total_tokens, batch, H, D, _pv(pv_mode)))


# ----------------------------------------------------------------- forward --

def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
             sm_scale: Optional[float] = None, pv_mode: str = "fp16",
             out_dtype: Optional[torch.dtype] = None, out: Optional[torch.Tensor] = None,
             workspace: Optional[Workspace] = None, qk_gran: str = "block",
             sq_chunk_blocks: Optional[int] = None) -> torch.Tensor:
    """SageAttention forward over dense [B, H, N, D] fp16/bf16 tensors.

    k and v may have fewer heads than q ([B, Hkv, N, D], H a multiple of Hkv):
    grouped-query attention, query head h reading key/value head h // (H // Hkv).
    qk_gran: "block" (one Q/K delta per 128 tokens), "token" (one per token) or
    "block_sq" (per block, with each Q block smoothed by its channel mean).
    sq_chunk_blocks ("block_sq"): query blocks whose mean term the workspace
    holds at a time (even, or at least all of them); by default as many as fit
    256 MiB.  The output does not depend on it.
    """
    _need_cuda_contig(q, k, v)
    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape:
        raise ValueError("q must be [B, H, N, D] and k, v one [B, Hkv, N, D] shape")
    B, H, N, D = q.shape
    Hkv = k.shape[1]
    if (k.shape[0], k.shape[2], k.shape[3]) != (B, N, D) or Hkv < 1 or H % Hkv:
        raise ValueError("k, v must be [B, Hkv, N, D] with Hkv dividing H")
    if k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must share one dtype")
    od = out_dtype or q.dtype
    if out is None:
        out = torch.empty((B, H, N, D), dtype=od, device=q.device)
    _need_cuda_contig(out)
    mode = _pv(pv_mode)
    scale = float(sm_scale) if sm_scale else 0.0
    lib = _lib.load()
    gran = _gran(qk_gran)
    if gran:
        if gran == 2 and sq_chunk_blocks is not None:
            nbytes = int(lib.sage_workspace_bytes_sq(B, H, Hkv, N, D, mode, int(sq_chunk_blocks)))
            if nbytes == 0:
                raise ValueError("sq_chunk_blocks must be even or at least ceil(N/128)")
        else:
            nbytes = int(lib.sage_workspace_bytes_ex(B, H, Hkv, N, D, mode, gran))
        ws = _workspace(q.device, nbytes, workspace)
        # with a chosen chunk, exactly the bytes that size it (a cached
        # workspace may be larger, and the call would hold more blocks)
        _check(lib.sage_attn_fwd_ex(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q.dtype),
            _dtype_code(out.dtype, True), B, H, Hkv, N, D, int(bool(causal)), scale, mode, gran,
            ws.ptr, nbytes if sq_chunk_blocks is not None else ws.nbytes, _stream(q.device)),
            "sage_attn_fwd_ex")
    elif Hkv == H:
        ws = _workspace(q.device, workspace_bytes(B, H, N, D, pv_mode), workspace)
        _check(lib.sage_attn_fwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q.dtype),
            _dtype_code(out.dtype, True), B, H, N, D, int(bool(causal)), scale, mode, ws.ptr,
            ws.nbytes, _stream(q.device)), "sage_attn_fwd")
    else:
        ws = _workspace(q.device, workspace_bytes_gqa(B, H, Hkv, N, D, pv_mode), workspace)
        _check(lib.sage_attn_fwd_gqa(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q.dtype),
            _dtype_code(out.dtype, True), B, H, Hkv, N, D, int(bool(causal)), scale, mode,
            ws.ptr, ws.nbytes, _stream(q.device)), "sage_attn_fwd_gqa")
    return out


# ---------------------------------------------------- host-resident inputs --

_host_state: dict = {}


def dense_host_pieces(B: int, Hkv: int, per: int) -> list:
    """Pieces (batch, first key/value head, heads) of attn_fwd_host: `per`
    heads each, except that the job's first and last pieces are cut down to
    one head -- the first upload is what the pipeline waits for before any
    work, the last piece's work and download are what it waits for after the
    last upload."""
    pieces = [(b, h0, min(per, Hkv - h0)) for b in range(B) for h0 in range(0, Hkv, per)]
    if pieces[0][2] > 1:
        b, h0, nh = pieces[0]
        pieces[0:1] = [(b, h0, 1), (b, h0 + 1, nh - 1)]
    if pieces[-1][2] > 1:
        b, h0, nh = pieces[-1]
        pieces[-1:] = [(b, h0, nh - 1), (b, h0 + nh - 1, 1)]
    return pieces


def varlen_host_order(pieces: list, cu: list) -> list:
    """Order of attn_fwd_varlen_host's pieces (sequence ranges [a, b)): the one
    with the fewest tokens first and the next fewest last, for the same reason
    as dense_host_pieces.  Pieces are independent problems, each writing its
    own token range of the output, so any order gives the same result."""
    if len(pieces) <= 2:
        return list(pieces)
    order = sorted(range(len(pieces)), key=lambda i: cu[pieces[i][1]] - cu[pieces[i][0]])
    ends = {order[0], order[1]}
    return ([pieces[order[0]]] + [x for i, x in enumerate(pieces) if i not in ends]
            + [pieces[order[1]]])


def attn_fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, out: torch.Tensor,
                  causal: bool = False, sm_scale: Optional[float] = None, pv_mode: str = "fp16",
                  qk_gran: str = "block", device=None, chunks: int = 16,
                  slots: int = 3) -> torch.Tensor:
    """attn_fwd for dense tensors that live in (pinned) host memory, result
    written to the host tensor `out`.

    The problem is cut into about `chunks` pieces along (batch, key/value head
    group) -- independent problems, since every statistic of the method (K
    mean, deltas, V scales, softmax) is per (sequence, head) -- each with at
    least as many work items as the GPU has SMs.  Each piece is
    uploaded on a copy-in stream, computed on its slot's own stream with its
    own workspace, and downloaded on a copy-out stream; `slots` pieces are in
    flight.  So uploads, downloads and compute overlap, and a piece's kernels
    fill the SMs that the previous piece's last work items leave idle.  The
    result equals one attn_fwd over the whole input.  Returns `out`; the work
    is ordered before anything later on the current stream.
    """
    if q.is_cuda or k.is_cuda or v.is_cuda or out.is_cuda:
        raise ValueError("attn_fwd_host takes host tensors")
    if q.dim() != 4 or k.dim() != 4 or v.shape != k.shape or out.shape != q.shape:
        raise ValueError("q, out must be [B, H, N, D] and k, v one [B, Hkv, N, D] shape")
    if not all(t.is_contiguous() for t in (q, k, v, out)):
        raise ValueError("tensors must be contiguous")
    if slots < 2:
        raise ValueError("slots must be at least 2")
    B, H, N, D = q.shape
    Hkv = k.shape[1]
    if H % Hkv:
        raise ValueError("Hkv must divide H")
    g = H // Hkv
    dev = torch.device(device if device is not None else "cuda")
    # key/value heads per piece: a divisor of Hkv, about `chunks` pieces in
    # all, but at least one full wave of the attention kernel's work items
    # (pairs of 128-row query tiles) per piece
    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    items_per_kv_head = g * ((N + 2 * BLOCK - 1) // (2 * BLOCK))
    per = max(1, (B * Hkv) // max(1, chunks), -(-sms // items_per_kv_head))
    per = min(per, Hkv)
    while Hkv % per:
        per += 1
    pieces = dense_host_pieces(B, Hkv, per)
    key = (dev.index, q.dtype, out.dtype, per * g, per, N, D, slots, pv_mode, qk_gran)
    st = _host_state.get(key)
    if st is None:
        e = dict(dtype=q.dtype, device=dev)
        nbytes = int(_lib.load().sage_workspace_bytes_ex(1, per * g, per, N, D, _pv(pv_mode),
                                                         _gran(qk_gran)))
        st = _host_state[key] = dict(
            q=[torch.empty((1, per * g, N, D), **e) for _ in range(slots)],
            k=[torch.empty((1, per, N, D), **e) for _ in range(slots)],
            v=[torch.empty((1, per, N, D), **e) for _ in range(slots)],
            o=[torch.empty((1, per * g, N, D), dtype=out.dtype, device=dev) for _ in range(slots)],
            ws=[Workspace(nbytes, dev) for _ in range(slots)],
            comp=[torch.cuda.Stream(dev) for _ in range(slots)],
            s_in=torch.cuda.Stream(dev), s_out=torch.cuda.Stream(dev),
            ev=[[torch.cuda.Event() for _ in range(3)] for _ in range(slots)])
    cur = torch.cuda.current_stream(dev)
    s_in, s_out, comp = st["s_in"], st["s_out"], st["comp"]
    for s_ in (s_in, s_out, *comp):  # ordered after everything enqueued before the call
        s_.wait_stream(cur)
    for c, (b, h0, nh) in enumerate(pieces):
        slot = c % slots
        ev_in, ev_comp, ev_out = st["ev"][slot]
        hq = slice(h0 * g, (h0 + nh) * g)
        hk = slice(h0, h0 + nh)
        # the slot's buffers hold `per` heads; a piece uses the leading nh
        sq, sk, sv, so = (st[n][slot][:, :w] for n, w in
                          (("q", nh * g), ("k", nh), ("v", nh), ("o", nh * g)))
        with torch.cuda.stream(s_in):
            if c >= slots:
                s_in.wait_event(ev_comp)          # the slot's inputs were consumed
            sq[0].copy_(q[b, hq], non_blocking=True)
            sk[0].copy_(k[b, hk], non_blocking=True)
            sv[0].copy_(v[b, hk], non_blocking=True)
            ev_in.record(s_in)
        cs = comp[slot]
        cs.wait_event(ev_in)
        if c >= slots:
            cs.wait_event(ev_out)                 # the slot's last result was downloaded
        with torch.cuda.stream(cs):
            attn_fwd(sq, sk, sv, causal=causal, sm_scale=sm_scale, pv_mode=pv_mode, out=so,
                     workspace=st["ws"][slot], qk_gran=qk_gran)
            ev_comp.record(cs)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp)
            out[b, hq].copy_(so[0], non_blocking=True)
            ev_out.record(s_out)
    for s_ in (s_out, s_in, *comp):
        cur.wait_stream(s_)
    return out


def attn_fwd_varlen_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                         cu_seqlens: torch.Tensor, out: torch.Tensor, causal: bool = False,
                         sm_scale: Optional[float] = None, pv_mode: str = "fp16",
                         qk_gran: str = "block", device=None, chunks: int = 8,
                         slots: int = 3) -> torch.Tensor:
    """attn_fwd_varlen for packed tensors that live in (pinned) host memory,
    result written to the host tensor `out` ([T, H, D]).

    The batch is cut into about `chunks` pieces of consecutive sequences with
    about equal token counts: each piece is a contiguous range of rows and an
    independent packed problem (every statistic of the method is per
    sequence), with its own cu_seqlens.  Pieces are uploaded on a copy-in
    stream, computed on their slot's stream with the slot's workspace and
    downloaded on a copy-out stream, `slots` pieces in flight.  The result
    equals one attn_fwd_varlen over the whole batch.  cu_seqlens: host int32
    [batch + 1].  Returns `out`; the work is ordered before anything later on
    the current stream.
    """
    if any(t.is_cuda for t in (q, k, v, out, cu_seqlens)):
        raise ValueError("attn_fwd_varlen_host takes host tensors")
    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape or out.shape != q.shape:
        raise ValueError("q, out must be [T, H, D] and k, v one [T, Hkv, D] shape")
    if not all(t.is_contiguous() for t in (q, k, v, out)):
        raise ValueError("tensors must be contiguous")
    if cu_seqlens.dtype != torch.int32 or slots < 2:
        raise ValueError("cu_seqlens must be int32 and slots at least 2")
    T, H, D = q.shape
    Hkv = k.shape[1]
    cu = [int(x) for x in cu_seqlens.tolist()]
    batch = len(cu) - 1
    if batch < 1 or cu[0] != 0 or cu[-1] != T or any(b < a for a, b in zip(cu, cu[1:])):
        raise ValueError("cu_seqlens must rise from 0 to T")
    dev = torch.device(device if device is not None else "cuda")
    # consecutive sequences, about T / chunks tokens per piece
    pieces, s0 = [], 0
    for c in range(max(1, chunks)):
        goal = T * (c + 1) / max(1, chunks)
        s1 = s0
        while s1 < batch and (s1 == s0 or cu[s1 + 1] <= goal or c == chunks - 1):
            s1 += 1
        if s1 > s0:
            pieces.append((s0, s1))
        s0 = s1
        if s0 >= batch:
            break
    if s0 < batch:
        pieces.append((s0, batch))
    pieces = varlen_host_order(pieces, cu)
    tmax = max(cu[b] - cu[a] for a, b in pieces)
    bmax = max(b - a for a, b in pieces)
    key = ("varlen", dev.index, q.dtype, out.dtype, H, Hkv, D, tmax, bmax, slots)
    st = _host_state.get(key)
    if st is None:
        e = dict(dtype=q.dtype, device=dev)
        st = _host_state[key] = dict(
            q=[torch.empty((tmax, H, D), **e) for _ in range(slots)],
            k=[torch.empty((tmax, Hkv, D), **e) for _ in range(slots)],
            v=[torch.empty((tmax, Hkv, D), **e) for _ in range(slots)],
            o=[torch.empty((tmax, H, D), dtype=out.dtype, device=dev) for _ in range(slots)],
            ws=[Workspace(256, dev) for _ in range(slots)],
            comp=[torch.cuda.Stream(dev) for _ in range(slots)],
            s_in=torch.cuda.Stream(dev), s_out=torch.cuda.Stream(dev),
            ev=[[torch.cuda.Event() for _ in range(3)] for _ in range(slots)])
    cur = torch.cuda.current_stream(dev)
    s_in, s_out, comp = st["s_in"], st["s_out"], st["comp"]
    for s_ in (s_in, s_out, *comp):  # ordered after everything enqueued before the call
        s_.wait_stream(cur)
    # every piece's own cu_seqlens (rebased to its first token), one upload
    offs, local = [], []
    for a, b in pieces:
        offs.append(len(local))
        local += [x - cu[a] for x in cu[a:b + 1]]
    with torch.cuda.stream(s_in):
        cu_d = torch.tensor(local, dtype=torch.int32).pin_memory().to(dev, non_blocking=True)
    for c, (a, b) in enumerate(pieces):
        slot = c % slots
        ev_in, ev_comp, ev_out = st["ev"][slot]
        t0, t1 = cu[a], cu[b]
        n = t1 - t0
        lens = [cu[i + 1] - cu[i] for i in range(a, b)]
        with torch.cuda.stream(s_in):
            if c >= slots:
                s_in.wait_event(ev_comp)          # the slot's inputs were consumed
            if n:
                st["q"][slot][:n].copy_(q[t0:t1], non_blocking=True)
                st["k"][slot][:n].copy_(k[t0:t1], non_blocking=True)
                st["v"][slot][:n].copy_(v[t0:t1], non_blocking=True)
            ev_in.record(s_in)
        cs = comp[slot]
        cs.wait_event(ev_in)
        if c >= slots:
            cs.wait_event(ev_out)                 # the slot's last result was downloaded
        with torch.cuda.stream(cs):
            if n:
                attn_fwd_varlen(st["q"][slot][:n], st["k"][slot][:n], st["v"][slot][:n],
                                cu_d[offs[c]:offs[c] + b - a + 1], max(lens), causal=causal,
                                sm_scale=sm_scale, pv_mode=pv_mode, out=st["o"][slot][:n],
                                workspace=st["ws"][slot], qk_gran=qk_gran)
            ev_comp.record(cs)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp)
            if n:
                out[t0:t1].copy_(st["o"][slot][:n], non_blocking=True)
            ev_out.record(s_out)
    for s_ in (s_out, s_in, *comp):
        cur.wait_stream(s_)
    cu_d.record_stream(cur)
    for cs in comp:
        cu_d.record_stream(cs)
    return out


def attn_fwd_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                    max_seqlen: int, causal: bool = False, sm_scale: Optional[float] = None,
                    pv_mode: str = "fp16", out_dtype: Optional[torch.dtype] = None,
                    out: Optional[torch.Tensor] = None,
                    workspace: Optional[Workspace] = None, qk_gran: str = "block") -> torch.Tensor:
    """SageAttention forward over packed [T, H, D] tensors with int32 cu_seqlens.
    k, v may be [T, Hkv, D] with Hkv dividing H (grouped-query attention);
    qk_gran: one Q/K delta per 128-token block ("block"), per token ("token"),
    or per block with Q smoothing ("block_sq")."""
    _need_cuda_contig(q, k, v, cu_seqlens)
    if q.dim() != 3 or k.dim() != 3 or v.shape != k.shape:
        raise ValueError("q must be [T, H, D] and k, v one [T, Hkv, D] shape")
    if cu_seqlens.dtype != torch.int32:
        raise ValueError("cu_seqlens must be int32")
    T, H, D = q.shape
    Hkv = k.shape[1]
    if (k.shape[0], k.shape[2]) != (T, D) or H % Hkv:
        raise ValueError("k, v must be [T, Hkv, D] with Hkv dividing H")
    batch = cu_seqlens.numel() - 1
    od = out_dtype or q.dtype
    if out is None:
        out = torch.empty((T, H, D), dtype=od, device=q.device)
    _need_cuda_contig(out)
    mode = _pv(pv_mode)
    lib = _lib.load()
    scale = float(sm_scale) if sm_scale else 0.0
    gran = _gran(qk_gran)
    if gran:
        if qk_gran == "block_sq":  # its workspace depends on max_seqlen
            nb = int(lib.sage_workspace_bytes_varlen_sq(T, batch, int(max_seqlen), H, Hkv, D, mode))
        else:
            nb = int(lib.sage_workspace_bytes_varlen_ex(T, batch, H, Hkv, D, mode, gran))
        ws = _workspace(q.device, nb, workspace)
        _check(lib.sage_attn_fwd_varlen_ex(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q.dtype),
            _dtype_code(out.dtype, True), _ptr(cu_seqlens), batch, int(max_seqlen), T, H, Hkv, D,
            int(bool(causal)), scale, mode, gran, ws.ptr, ws.nbytes, _stream(q.device)),
            "sage_attn_fwd_varlen_ex")
    elif Hkv == H:
        ws = _workspace(q.device, workspace_bytes_varlen(T, batch, H, D, pv_mode), workspace)
        _check(lib.sage_attn_fwd_varlen(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q.dtype),
            _dtype_code(out.dtype, True), _ptr(cu_seqlens), batch, int(max_seqlen), T, H, D,
            int(bool(causal)), scale, mode, ws.ptr, ws.nbytes, _stream(q.device)),
            "sage_attn_fwd_varlen")
    else:
        ws = _workspace(q.device, int(lib.sage_workspace_bytes_varlen_gqa(T, batch, H, Hkv, D,
                                                                          mode)), workspace)
        _check(lib.sage_attn_fwd_varlen_gqa(
            _ptr(q), _ptr(k), _ptr(v), _ptr(out), _dtype_code(q.dtype),
            _dtype_code(out.dtype, True), _ptr(cu_seqlens), batch, int(max_seqlen), T, H, Hkv, D,
            int(bool(causal)), scale, mode, ws.ptr, ws.nbytes, _stream(q.device)),
            "sage_attn_fwd_varlen_gqa")
    return out


# ---------------------------------------------------------------- stages --

QK_GRANS = {"block": 0, "token": 1, "block_sq": 2}


def _gran(g: str) -> int:
    if g not in QK_GRANS:
        raise ValueError(f"qk_gran must be one of {sorted(QK_GRANS)}")
    return QK_GRANS[g]


@dataclasses.dataclass
class Quantized:
    """Outputs of the smoothing + quantisation stage (all device tensors).
    Dense: q_codes [B, H, NP, D], k_codes [B, Hkv, NP, D]; deltas [.., NB]
    per 128-token block or [.., NP] per token (qk_gran).  Q smoothing
    ("block_sq") adds the Q block means q_mean [B, H, NB, D] and the per-key
    mean term q_bias [B, H, NB, NP], which depends on the attention call's
    causal flag and sm_scale (recorded in sq_causal, sq_sm_scale)."""
    q_codes: torch.Tensor
    q_scale: torch.Tensor
    k_codes: torch.Tensor
    k_scale: torch.Tensor
    k_mean: torch.Tensor
    v_codes: Optional[torch.Tensor]
    v_scale: Optional[torch.Tensor]
    pv_mode: str
    qk_gran: str = "block"
    q_mean: Optional[torch.Tensor] = None
    q_bias: Optional[torch.Tensor] = None
    sq_causal: bool = False
    sq_sm_scale: float = 0.0


def alloc_quantized(B: int, H: int, N: int, D: int, pv_mode: str, device,
                    Hkv: Optional[int] = None, qk_gran: str = "block") -> Quantized:
    NB = (N + BLOCK - 1) // BLOCK
    _gran(qk_gran)
    NS = NB * BLOCK if qk_gran == "token" else NB
    Hk = Hkv or H
    fp8 = pv_mode == "fp8"
    sq = qk_gran == "block_sq"
    e = dict(device=device)
    return Quantized(
        torch.empty((B, H, NB * BLOCK, D), dtype=torch.int8, **e),
        torch.empty((B, H, NS), dtype=torch.float32, **e),
        torch.empty((B, Hk, NB * BLOCK, D), dtype=torch.int8, **e),
        torch.empty((B, Hk, NS), dtype=torch.float32, **e),
        torch.empty((B, Hk, D), dtype=torch.float32, **e),
        torch.empty((B, Hk, N, D), dtype=torch.uint8, **e) if fp8 else None,
        torch.empty((B, Hk, D), dtype=torch.float32, **e) if fp8 else None,
        pv_mode, qk_gran,
        torch.empty((B, H, NB, D), dtype=torch.float32, **e) if sq else None,
        torch.empty((B, H, NB, NB * BLOCK), dtype=torch.float32, **e) if sq else None)


def quantize(q: torch.Tensor, k: torch.Tensor, v: Optional[torch.Tensor] = None,
             pv_mode: str = "fp16", qz: Optional[Quantized] = None,
             workspace: Optional[Workspace] = None, qk_gran: str = "block",
             causal: bool = False, sm_scale: Optional[float] = None) -> Quantized:
    """Stage 1 (K smoothing, INT8 Q/K per block or per token, FP8 V) of a dense
    problem; k, v may have fewer heads than q (grouped-query).  With
    qk_gran "block_sq" Q is smoothed too, and causal / sm_scale must be those
    of the attention call (the per-key mean term is scaled and masked here)."""
    _need_cuda_contig(q, k)
    B, H, N, D = q.shape
    Hkv = k.shape[1]
    mode = _pv(pv_mode)
    gran = _gran(qk_gran)
    if mode == 1:
        if v is None:
            raise ValueError("FP8 P.V needs v")
        _need_cuda_contig(v)
    qz = qz or alloc_quantized(B, H, N, D, pv_mode, q.device, Hkv, qk_gran)
    ws = _workspace(q.device, int(_lib.load().sage_scratch_bytes(B, H, D)), workspace)
    if qk_gran == "block_sq":
        scale = float(sm_scale) if sm_scale else 0.0
        _check(_lib.load().sage_quantize_sq(
            _ptr(q), _ptr(k), _ptr(v) if mode == 1 else None, _dtype_code(q.dtype), B, H, Hkv, N,
            D, mode, int(bool(causal)), scale, _ptr(qz.q_codes), _ptr(qz.q_scale),
            _ptr(qz.q_mean), _ptr(qz.k_codes), _ptr(qz.k_scale), _ptr(qz.k_mean),
            _ptr(qz.v_codes), _ptr(qz.v_scale), _ptr(qz.q_bias), ws.ptr, ws.nbytes,
            _stream(q.device)), "sage_quantize_sq")
        qz.sq_causal, qz.sq_sm_scale = bool(causal), scale
        return qz
    _check(_lib.load().sage_quantize_ex(
        _ptr(q), _ptr(k), _ptr(v) if mode == 1 else None, _dtype_code(q.dtype), B, H, Hkv, N, D,
        mode, gran, _ptr(qz.q_codes), _ptr(qz.q_scale), _ptr(qz.k_codes), _ptr(qz.k_scale),
        _ptr(qz.k_mean), _ptr(qz.v_codes), _ptr(qz.v_scale), ws.ptr, ws.nbytes,
        _stream(q.device)), "sage_quantize_ex")
    return qz


def quant_qk(q: torch.Tensor, k: torch.Tensor,
             workspace: Optional[Workspace] = None) -> Quantized:
    """K smoothing and per-block INT8 quantisation of q and k alone (dense,
    k with the heads of q), through sage_quant_qk."""
    _need_cuda_contig(q, k)
    B, H, N, D = q.shape
    qz = alloc_quantized(B, H, N, D, "fp16", q.device)
    ws = _workspace(q.device, int(_lib.load().sage_scratch_bytes(B, H, D)), workspace)
    _check(_lib.load().sage_quant_qk(
        _ptr(q), _ptr(k), _dtype_code(q.dtype), B, H, N, D, _ptr(qz.q_codes), _ptr(qz.q_scale),
        _ptr(qz.k_codes), _ptr(qz.k_scale), _ptr(qz.k_mean), ws.ptr, ws.nbytes,
        _stream(q.device)), "sage_quant_qk")
    return qz


def attn_quantized_dump_s(qz: Quantized, v: torch.Tensor, causal: bool = False,
                          sm_scale: Optional[float] = None,
                          fill: int = -2 ** 31) -> tuple[torch.Tensor, torch.Tensor]:
    """Stage 2 of a dense problem (per-block deltas; fp16 V or FP8 P.V) with
    the attention kernel's own int32 QK^T scores stored as it computes them.
    Returns (out fp32 [B, H, N, D], S int32 [B*H, NP, NP]); entries of S the
    kernel does not visit keep `fill`."""
    _need_cuda_contig(v)
    B, H, NP, D = qz.q_codes.shape
    N = v.shape[2]
    out = torch.empty((B, H, N, D), dtype=torch.float32, device=v.device)
    s = torch.full((B * H, NP, NP), fill, dtype=torch.int32, device=v.device)
    ws = _workspace(v.device, int(_lib.load().sage_scratch_bytes(B, H, D)), None)
    _check(_lib.load().sage_attn_quantized_dump_s(
        _ptr(qz.q_codes), _ptr(qz.q_scale), _ptr(qz.k_codes), _ptr(qz.k_scale), _ptr(v),
        _ptr(qz.v_codes), _ptr(qz.v_scale), _ptr(out), _dtype_code(v.dtype),
        _dtype_code(out.dtype, True), B, H, N, D, int(bool(causal)),
        float(sm_scale) if sm_scale else 0.0, _pv(qz.pv_mode), _ptr(s), ws.ptr, ws.nbytes,
        _stream(v.device)), "sage_attn_quantized_dump_s")
    return out, s


def attn_quantized(qz: Quantized, v: torch.Tensor, causal: bool = False,
                   sm_scale: Optional[float] = None, out_dtype: Optional[torch.dtype] = None,
                   out: Optional[torch.Tensor] = None,
                   workspace: Optional[Workspace] = None) -> torch.Tensor:
    """Stage 2 (fused INT8 QK^T, online softmax, P.V) from stage-1 outputs."""
    _need_cuda_contig(v)
    B, H, NP, D = qz.q_codes.shape
    Hkv, N = v.shape[1], v.shape[2]
    mode = _pv(qz.pv_mode)
    od = out_dtype or v.dtype
    if out is None:
        out = torch.empty((B, H, N, D), dtype=od, device=v.device)
    ws = _workspace(v.device, int(_lib.load().sage_scratch_bytes(B, H, D)), workspace)
    if qz.qk_gran == "block_sq":
        scale = float(sm_scale) if sm_scale else 0.0
        if bool(causal) != qz.sq_causal or scale != qz.sq_sm_scale:
            raise ValueError("Q smoothing's mean term was built for another causal / sm_scale")
        _check(_lib.load().sage_attn_quantized_sq(
            _ptr(qz.q_codes), _ptr(qz.q_scale), _ptr(qz.k_codes), _ptr(qz.k_scale),
            _ptr(qz.q_bias), _ptr(v), _ptr(qz.v_codes), _ptr(qz.v_scale), _ptr(out),
            _dtype_code(v.dtype), _dtype_code(out.dtype, True), B, H, Hkv, N, D,
            int(bool(causal)), scale, mode, ws.ptr, ws.nbytes, _stream(v.device)),
            "sage_attn_quantized_sq")
        return out
    _check(_lib.load().sage_attn_quantized_ex(
        _ptr(qz.q_codes), _ptr(qz.q_scale), _ptr(qz.k_codes), _ptr(qz.k_scale), _ptr(v),
        _ptr(qz.v_codes), _ptr(qz.v_scale), _ptr(out), _dtype_code(v.dtype),
        _dtype_code(out.dtype, True), B, H, Hkv, N, D, int(bool(causal)),
        float(sm_scale) if sm_scale else 0.0, mode, _gran(qz.qk_gran), ws.ptr, ws.nbytes,
        _stream(v.device)), "sage_attn_quantized_ex")
    return out


def quantize_varlen(q: torch.Tensor, k: torch.Tensor, v: Optional[torch.Tensor],
                    cu_seqlens: torch.Tensor, max_seqlen: int, pv_mode: str = "fp16",
                    workspace: Optional[Workspace] = None) -> Quantized:
    """Stage 1 of a packed varlen batch; code layout [H, TBmax*128, D]."""
    _need_cuda_contig(q, k, cu_seqlens)
    T, H, D = q.shape
    batch = cu_seqlens.numel() - 1
    mode = _pv(pv_mode)
    TB = (T + (BLOCK - 1) * batch) // BLOCK
    e = dict(device=q.device)
    fp8 = mode == 1
    qz = Quantized(
        torch.empty((H, TB * BLOCK, D), dtype=torch.int8, **e),
        torch.empty((H, TB), dtype=torch.float32, **e),
        torch.empty((H, TB * BLOCK, D), dtype=torch.int8, **e),
        torch.empty((H, TB), dtype=torch.float32, **e),
        torch.empty((batch, H, D), dtype=torch.float32, **e),
        torch.empty((T, H, D), dtype=torch.uint8, **e) if fp8 else None,
        torch.empty((batch, H, D), dtype=torch.float32, **e) if fp8 else None,
        pv_mode)
    ws = _workspace(q.device, workspace_bytes_varlen(T, batch, H, D, pv_mode), workspace)
    _check(_lib.load().sage_quantize_varlen(
        _ptr(q), _ptr(k), _ptr(v) if fp8 else None, _dtype_code(q.dtype), _ptr(cu_seqlens), batch,
        int(max_seqlen), T, H, D, mode, _ptr(qz.q_codes), _ptr(qz.q_scale), _ptr(qz.k_codes),
        _ptr(qz.k_scale), _ptr(qz.k_mean), _ptr(qz.v_codes), _ptr(qz.v_scale), ws.ptr, ws.nbytes,
        _stream(q.device)), "sage_quantize_varlen")
    return qz


def qk_int8_tiles(q_codes: torch.Tensor, k_codes: torch.Tensor,
                  tiles: Sequence[tuple[int, int, int]],
                  workspace: Optional[Workspace] = None) -> torch.Tensor:
    """int32 QK^T tiles (bh, I, J) of dense [B, H, NP, D] code arrays, through the
    attention kernel's TMA + tcgen05 INT8 path.  Returns [n, 128, 128]."""
    _need_cuda_contig(q_codes, k_codes)
    B, H, NP, D = q_codes.shape
    flat = [int(x) for t in tiles for x in t]
    arr = (ctypes.c_int32 * len(flat))(*flat)
    out = torch.empty((len(tiles), BLOCK, BLOCK), dtype=torch.int32, device=q_codes.device)
    ws = _workspace(q_codes.device, 256 + 256 * (1 + len(flat) * 4 // 256), workspace)
    _check(_lib.load().sage_qk_int8_tiles(
        _ptr(q_codes), _ptr(k_codes), B * H, NP, D, ctypes.cast(arr, ctypes.c_void_p),
        len(tiles), _ptr(out), ws.ptr, ws.nbytes, _stream(q_codes.device)), "sage_qk_int8_tiles")
    return out


# ------------------------------------------------ accuracy-driven P.V mode --
#
# "SageAttention v1/v2/v2++/v3 overview", SageAttention v1, adaptive
# quantisation: the faster kernel variant is tested layer by layer on several
# inputs, and a layer uses it only where its cosine similarity to
# full-precision attention is above 99.8 % (the lowest similarity of the
# accurate variant); the other layers keep the accurate variant.  Here the
# faster variant is FP8 P.V and the accurate one 16-bit P.V.

PV_COSINE_THRESHOLD = 0.998


def attn_ref_rows(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, rows,
                  causal: bool = False, sm_scale: Optional[float] = None) -> torch.Tensor:
    """Full-precision (fp32, unquantised) attention for the (b, h, i) query rows
    `rows` of dense [B, H, N, D] q over [B, Hkv, N, D] k, v; returns [n, D] fp32."""
    _need_cuda_contig(q, k, v)
    B, H, N, D = q.shape
    r = torch.as_tensor(rows, dtype=torch.int32).reshape(-1, 3).contiguous().to(q.device)
    out = torch.empty((r.shape[0], D), dtype=torch.float32, device=q.device)
    _check(_lib.load().sage_attn_ref_rows(
        _ptr(q), _ptr(k), _ptr(v), _dtype_code(q.dtype), B, H, k.shape[1], N, D,
        int(bool(causal)), float(sm_scale) if sm_scale else 0.0, _ptr(r), int(r.shape[0]),
        _ptr(out), _stream(q.device)), "sage_attn_ref_rows")
    return out


def cosine_similarity(a: torch.Tensor, b: torch.Tensor) -> float:
    """Cosine similarity of two tensors taken as flat vectors (host, float64)."""
    x = a.detach().double().cpu().flatten()
    y = b.detach().double().cpu().flatten()
    return float((x @ y) / (x.norm() * y.norm()))


def choose_pv_mode(cos_fp8: float, threshold: float = PV_COSINE_THRESHOLD) -> str:
    """FP8 P.V where its cosine similarity to full precision is above the
    threshold, 16-bit P.V otherwise."""
    return "fp8" if cos_fp8 > threshold else "fp16"


def sample_query_rows(B: int, H: int, N: int, n_rows: int, seed: int = 0) -> list:
    """Seeded (b, h, i) rows: the first and last row of every head plus uniform draws."""
    g = torch.Generator().manual_seed(seed)
    picks = {(b, h, i) for b in range(B) for h in range(H) for i in (0, N - 1)}
    total = B * H * N
    while len(picks) < min(max(n_rows, len(picks)), total):
        u = int(torch.randint(0, total, (1,), generator=g))
        picks.add((u // (H * N), (u // N) % H, u % N))
    return sorted(picks)


def pv_mode_similarity(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, causal: bool = False,
                       sm_scale: Optional[float] = None, n_rows: int = 256,
                       seed: int = 0) -> dict:
    """Cosine similarity to full-precision attention of both P.V modes on
    sampled query rows of one input."""
    B, H, N, D = q.shape
    rows = sample_query_rows(B, H, N, n_rows, seed)
    ref = attn_ref_rows(q, k, v, rows, causal, sm_scale)
    idx = torch.tensor(rows, dtype=torch.long, device=q.device)
    res = {}
    for mode in ("fp16", "fp8"):
        o = attn_fwd(q, k, v, causal=causal, sm_scale=sm_scale, pv_mode=mode,
                     out_dtype=torch.float32)
        res[mode] = cosine_similarity(o[idx[:, 0], idx[:, 1], idx[:, 2]], ref)
    return res


def calibrate_pv_modes(layers: dict, threshold: float = PV_COSINE_THRESHOLD,
                       measure=pv_mode_similarity) -> dict:
    """Per-layer P.V mode from sample inputs: `layers` maps a layer name to a
    list of (q, k, v, causal) inputs seen at that layer.  A layer gets FP8 P.V
    only if its lowest FP8 similarity over the inputs is above the threshold.
    Returns {name: (mode, lowest FP8 similarity, lowest 16-bit similarity)}."""
    out = {}
    for name, inputs in layers.items():
        sims = [measure(q, k, v, causal) for (q, k, v, causal) in inputs]
        lo8 = min(s["fp8"] for s in sims)
        lo16 = min(s["fp16"] for s in sims)
        out[name] = (choose_pv_mode(lo8, threshold), lo8, lo16)
    return out


def sync_status(workspace: Optional[Workspace] = None, device=None) -> None:
    """Synchronise and raise if any call on the workspace recorded a device error."""
    if workspace is None:
        dev = torch.device(device) if device is not None else torch.device("cuda")
        key = dev.index if dev.index is not None else torch.cuda.current_device()
        workspace = _default_ws.get(key)
        if workspace is None:
            return
    workspace.sync_status()


# --------------------------------------------------------- SDPA-style shim --

def sageattn(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, attn_mask=None,
             dropout_p: float = 0.0, is_causal: bool = False, scale: Optional[float] = None,
             pv_mode: str = "fp16", qk_gran: str = "block") -> torch.Tensor:
    """Drop-in for scaled_dot_product_attention on [B, H, N, D] fp16/bf16 inputs.

    Arbitrary masks and dropout are not part of the method; passing them raises
    SageError(SAGE_ERR_UNSUPPORTED).  Non-contiguous inputs (e.g. the
    transpose(1, 2) views of a projection output) are made contiguous first.
    k, v with fewer heads than q are grouped-query attention (no repeat_kv
    needed).
    """
    if attn_mask is not None or dropout_p:
        raise SageError(2, "sageattn: attn_mask / dropout_p")
    q, k, v = (t if t.is_contiguous() else t.contiguous() for t in (q, k, v))
    return attn_fwd(q, k, v, causal=is_causal, sm_scale=scale, pv_mode=pv_mode, qk_gran=qk_gran)


# The entry-point names of the SageAttention guide's API list ("SageAttention
# complete guide", advanced features: sageattn, sageattn_qk_int8_pv_fp8_cuda,
# sageattn_varlen), for callers switching over.  Each is argument marshalling
# around attn_fwd / attn_fwd_varlen; every step runs in this library's kernels.

def sageattn_qk_int8_pv_fp16_cuda(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                  is_causal: bool = False, sm_scale: Optional[float] = None,
                                  qk_gran: str = "block") -> torch.Tensor:
    """INT8 QK^T, 16-bit P.V with fp32 accumulation, [B, H, N, D] inputs."""
    q, k, v = (t if t.is_contiguous() else t.contiguous() for t in (q, k, v))
    return attn_fwd(q, k, v, causal=is_causal, sm_scale=sm_scale, pv_mode="fp16", qk_gran=qk_gran)


PV_ACCUM_DTYPES = ("fp32+fp32", "fp32")


def sageattn_qk_int8_pv_fp8_cuda(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor,
                                 is_causal: bool = False, sm_scale: Optional[float] = None,
                                 qk_gran: str = "block",
                                 pv_accum_dtype: str = "fp32+fp32") -> torch.Tensor:
    """INT8 QK^T, FP8 P.V with two-level fp32 accumulation (each 64-key tile's
    partial flushed into an fp32 accumulator).  pv_accum_dtype names that
    accumulation ("fp32+fp32"; "fp32" is taken as the same); other
    accumulation types are not implemented (SageError(SAGE_ERR_UNSUPPORTED))."""
    if pv_accum_dtype not in PV_ACCUM_DTYPES:
        raise SageError(2, f"pv_accum_dtype {pv_accum_dtype!r}")
    q, k, v = (t if t.is_contiguous() else t.contiguous() for t in (q, k, v))
    return attn_fwd(q, k, v, causal=is_causal, sm_scale=sm_scale, pv_mode="fp8", qk_gran=qk_gran)


def sageattn_varlen(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cu_seqlens: torch.Tensor,
                    max_seqlen: int, is_causal: bool = False, sm_scale: Optional[float] = None,
                    pv_mode: str = "fp16", qk_gran: str = "block") -> torch.Tensor:
    """Packed [T, H, D] sequences with int32 cu_seqlens (see attn_fwd_varlen)."""
    return attn_fwd_varlen(q, k, v, cu_seqlens, max_seqlen, causal=is_causal, sm_scale=sm_scale,
                           pv_mode=pv_mode, qk_gran=qk_gran)


def default_sm_scale(D: int) -> float:
    return 1.0 / math.sqrt(D)
