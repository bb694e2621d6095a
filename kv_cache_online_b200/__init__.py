"""kv_cache_online_b200 -- B200 (sm_100a) hot path of iS-KV online low-rank KV-cache compression.

Thin Python binding over ``libiskv.so`` (C ABI in ``include/iskv.h``). PyTorch provides device
memory and streams; every step of the fold, re-orthogonalisation, reconstruction and prompt-block
selection runs in the library's CUDA kernels. There is no CPU or PyTorch fallback: if the library is
missing, every call raises.

Sources: "iS-KV reading notes" (zhongzhuzhou.org), Sections 3-5 and Algorithms 1-3.
"""

from __future__ import annotations

import ctypes
import math

import torch

from . import _lib
from ._lib import ISKV_BF16, ISKV_F16, ISKV_F32, IskvError, IskvExactTable, IskvLowRank  # noqa: F401

_DT = {torch.float32: ISKV_F32, torch.bfloat16: ISKV_BF16, torch.float16: ISKV_F16}
_TD = {ISKV_F32: torch.float32, ISKV_BF16: torch.bfloat16, ISKV_F16: torch.float16}


def _dt(t: torch.Tensor) -> int:
    try:
        return _DT[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported dtype {t.dtype}; use float32, bfloat16 or float16") from None


def _stream(stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t):
    return None if t is None else t.data_ptr()


def _need_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("all tensors must live on a CUDA device")


class Workspace:
    """A reusable, 256-byte aligned device byte buffer grown on demand."""

    def __init__(self, device=None):
        self.device = device
        self.buf = None

    def get(self, nbytes: int) -> torch.Tensor:
        nbytes = max(int(nbytes), 256)
        if self.buf is None or self.buf.numel() < nbytes:
            self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=self.device)
        off = (-self.buf.data_ptr()) % 256
        return self.buf[off:off + nbytes]


_default_ws = {}


def _ws(device, nbytes):
    key = (str(device), "ws")
    w = _default_ws.get(key)
    if w is None:
        w = _default_ws[key] = Workspace(device)
    return w.get(nbytes)


class LowRankHistory:
    """One compressed history (a (sequence, layer, K|V) path): ``U diag(sigma) B^T`` with the
    original token position of every compressed row (Section 2.2 and Section 3.2).

    Device tensors: ``U`` (n_cap, r_max), ``sigma`` (r_max,) float32, ``B`` (d, r_max), ``pos``
    (n_cap,) int32, ``meta`` (4,) int64 = {k, n, folds since reorth, status bits}.
    """

    def __init__(self, d: int, r_max: int, n_cap: int, storage=torch.bfloat16, device="cuda"):
        self.d, self.r_max, self.n_cap = int(d), int(r_max), int(n_cap)
        self.storage = storage
        self.U = torch.zeros(self.n_cap, self.r_max, dtype=storage, device=device)
        self.sigma = torch.zeros(self.r_max, dtype=torch.float32, device=device)
        self.B = torch.zeros(self.d, self.r_max, dtype=storage, device=device)
        self.pos = torch.zeros(max(self.n_cap, 1), dtype=torch.int32, device=device)
        self.meta = torch.zeros(4, dtype=torch.int64, device=device)

    @property
    def device(self):
        return self.U.device

    def handle(self) -> IskvLowRank:
        return IskvLowRank(self.d, self.r_max, self.n_cap, _DT[self.storage], 0, _ptr(self.U),
                           _ptr(self.sigma), _ptr(self.B), _ptr(self.pos), _ptr(self.meta))

    def status(self):
        """(k, n, folds since reorth, status bits); synchronises the device."""
        k, n, f, s = (ctypes.c_int64() for _ in range(4))
        h = self.handle()
        _lib.check(_lib.load().iskv_get_status(ctypes.byref(h), ctypes.byref(k), ctypes.byref(n),
                                               ctypes.byref(f), ctypes.byref(s)), "get_status")
        return k.value, n.value, f.value, s.value

    def reset(self, stream=None):
        h = self.handle()
        _lib.check(_lib.load().iskv_reset(ctypes.byref(h), _stream(stream)), "reset")


def _handles(hists):
    arr = (IskvLowRank * len(hists))()
    for i, h in enumerate(hists):
        arr[i] = h.handle()
    return arr


def fold_workspace_size(count, d, r_max, b) -> int:
    return int(_lib.load().iskv_fold_workspace_size(count, d, r_max, b))


def fold_block_batched(hists, Fs, f_poss, tau_rel: float = 0.0, ws=None, stream=None,
                       factors_ready=None):
    """Algorithm 2 for every history in ``hists`` (one pending block each), in one launch set.
    ``factors_ready`` (a ``torch.cuda.Event``) lets the fold's read-only stages start at once and
    makes its factor-writing stages wait for the event (iskv_fold_block_batched_after)."""
    lib = _lib.load()
    n = len(hists)
    if n == 0:
        return
    b = int(Fs[0].shape[0])
    fdt = _dt(Fs[0])
    for F, p in zip(Fs, f_poss):
        _need_cuda(F, p)
        if F.shape != (b, hists[0].d) or _dt(F) != fdt or not F.is_contiguous():
            raise ValueError("every F must be a contiguous (b, d) tensor of one dtype")
        if p.dtype != torch.int32 or p.numel() != b or not p.is_contiguous():
            raise ValueError("f_pos must be a contiguous int32 tensor of b entries")
    need = lib.iskv_fold_workspace_size(n, hists[0].d, hists[0].r_max, b)
    w = ws if ws is not None else _ws(hists[0].device, need)
    hs = _handles(hists)
    Fp = (ctypes.c_void_p * n)(*[F.data_ptr() for F in Fs])
    Pp = (ctypes.c_void_p * n)(*[p.data_ptr() for p in f_poss])
    if factors_ready is None:
        _lib.check(lib.iskv_fold_block_batched(hs, n, Fp, fdt, b, Pp, float(tau_rel),
                                               w.data_ptr(), w.numel(), _stream(stream)),
                   "fold_block")
    else:
        _lib.check(lib.iskv_fold_block_batched_after(hs, n, Fp, fdt, b, Pp, float(tau_rel),
                                                     w.data_ptr(), w.numel(), _stream(stream),
                                                     factors_ready.cuda_event), "fold_block")


def fold_block(hist, F, f_pos, tau_rel: float = 0.0, ws=None, stream=None):
    """Algorithm 2: merge the pending block ``F`` (b, d) at positions ``f_pos`` into ``hist``."""
    fold_block_batched([hist], [F], [f_pos], tau_rel, ws, stream)


def reorth_workspace_size(count, d, r_max, n_cap) -> int:
    return int(_lib.load().iskv_reorth_workspace_size(count, d, r_max, n_cap))


def reorth(hists, ws=None, stream=None):
    """Section 4.4 re-orthogonalisation of every history in ``hists``."""
    if isinstance(hists, LowRankHistory):
        hists = [hists]
    lib = _lib.load()
    n = len(hists)
    need = lib.iskv_reorth_workspace_size(n, hists[0].d, hists[0].r_max, hists[0].n_cap)
    w = ws if ws is not None else _ws(hists[0].device, need)
    _lib.check(lib.iskv_reorth(_handles(hists), n, w.data_ptr(), w.numel(), _stream(stream)),
               "reorth")


def reconstruct_workspace_size(count, d, r_max) -> int:
    return int(_lib.load().iskv_reconstruct_workspace_size(count, d, r_max))


def reconstruct_batched(hists, exact_rows, exact_pos, n_total, n_heads, head_dim, rope,
                        theta=500000.0, outs=None, out_dtype=torch.bfloat16, ws=None, stream=None):
    """Algorithm 3 steps 7-8 for every history: dense (n_total, d) caches with compressed rows at
    their positions, exact rows copied, keys rotated (``rope[i]``)."""
    lib = _lib.load()
    n = len(hists)
    d = hists[0].d
    if isinstance(n_total, int):
        n_total = [n_total] * n
    if isinstance(rope, bool):
        rope = [rope] * n
    if outs is None:
        outs = [torch.empty(nt, d, dtype=out_dtype, device=h.device) for h, nt in zip(hists, n_total)]
    odt = _dt(outs[0])
    edt = ISKV_F32
    er, ep, ne = [], [], []
    for x, p in zip(exact_rows, exact_pos):
        if x is None or p is None or p.numel() == 0:
            er.append(None)
            ep.append(None)
            ne.append(0)
            continue
        _need_cuda(x, p)
        edt = _dt(x)
        if p.dtype != torch.int32 or x.shape != (p.numel(), d) or not x.is_contiguous():
            raise ValueError("exact rows must be (n_exact, d) contiguous with int32 positions")
        er.append(x.data_ptr())
        ep.append(p.data_ptr())
        ne.append(p.numel())
    need = lib.iskv_reconstruct_workspace_size(n, d, hists[0].r_max)
    w = ws if ws is not None else _ws(hists[0].device, need)
    _lib.check(lib.iskv_reconstruct_batched(
        _handles(hists), n, (ctypes.c_void_p * n)(*er), edt, (ctypes.c_void_p * n)(*ep),
        (ctypes.c_int64 * n)(*ne), (ctypes.c_int64 * n)(*n_total), n_heads, head_dim,
        (ctypes.c_int32 * n)(*[1 if r else 0 for r in rope]), float(theta),
        (ctypes.c_void_p * n)(*[o.data_ptr() for o in outs]), odt, w.data_ptr(), w.numel(),
        _stream(stream)), "reconstruct")
    return outs


def reconstruct(hist, exact_rows, exact_pos, n_total, n_heads, head_dim, rope, theta=500000.0,
                out=None, out_dtype=torch.bfloat16, ws=None, stream=None):
    """Single-history form of :func:`reconstruct_batched`."""
    return reconstruct_batched([hist], [exact_rows], [exact_pos], [n_total], n_heads, head_dim,
                               [rope], theta, None if out is None else [out], out_dtype, ws,
                               stream)[0]


def diagnostics(hists, n_exact=None, exact_bytes=2, ws=None, stream=None):
    """Section 5.1 eq. (12) and factor orthogonality for each history: device tensors
    ``(orth_u, orth_b)`` float64 (``||U^T U - I||_F``, ``||B^T B - I||_F`` over the current rank)
    and ``persistent_bytes`` int64."""
    lib = _lib.load()
    n = len(hists)
    dev = hists[0].device
    orth_u = torch.empty(n, dtype=torch.float64, device=dev)
    orth_b = torch.empty(n, dtype=torch.float64, device=dev)
    pbytes = torch.empty(n, dtype=torch.int64, device=dev)
    need = lib.iskv_diagnostics_workspace_size(n, hists[0].d, hists[0].r_max, hists[0].n_cap)
    w = ws if ws is not None else _ws(dev, need)
    ne = None if n_exact is None else (ctypes.c_int64 * n)(*[int(x) for x in n_exact])
    _lib.check(lib.iskv_diagnostics(_handles(hists), n, ne, int(exact_bytes), orth_u.data_ptr(),
                                    orth_b.data_ptr(), pbytes.data_ptr(), w.data_ptr(), w.numel(),
                                    _stream(stream)), "diagnostics")
    return orth_u, orth_b, pbytes


def attention_workspace_size(count, d, r_max, n_cap, n_total_max, n_q_heads) -> int:
    return int(_lib.load().iskv_attention_workspace_size(count, d, r_max, n_cap, n_total_max,
                                                         n_q_heads))


def _exact_arrays(rows, pos, d):
    ptr_r, ptr_p, cnt, dt = [], [], [], ISKV_F32
    for x, p in zip(rows, pos):
        if x is None or p is None or p.numel() == 0:
            ptr_r.append(None)
            ptr_p.append(None)
            cnt.append(0)
            continue
        _need_cuda(x, p)
        dt = _dt(x)
        if p.dtype != torch.int32 or x.shape != (p.numel(), d) or not x.is_contiguous():
            raise ValueError("exact rows must be (n_exact, d) contiguous with int32 positions")
        ptr_r.append(x.data_ptr())
        ptr_p.append(p.data_ptr())
        cnt.append(p.numel())
    return ptr_r, ptr_p, cnt, dt


def decode_attention_batched(k_hists, v_hists, k_exact, k_exact_pos, v_exact, v_exact_pos,
                             n_total, q, n_kv_heads, head_dim, theta=500000.0, scale=None,
                             outs=None, ws=None, stream=None):
    """Algorithm 3 steps 7-9 without the dense cache: one decode query ``q[i]`` (float32,
    ``(n_q_heads, head_dim)``, already rotated) per (K, V) history pair. Returns float32
    ``(n_q_heads, head_dim)`` outputs."""
    lib = _lib.load()
    n = len(k_hists)
    if len(v_hists) != n or len(q) != n:
        raise ValueError("one V history and one query per K history")
    d = k_hists[0].d
    if isinstance(n_total, int):
        n_total = [n_total] * n
    for x in q:
        _need_cuda(x)
        if x.dtype != torch.float32 or x.dim() != 2 or x.shape[1] != head_dim or not x.is_contiguous():
            raise ValueError("queries must be contiguous float32 (n_q_heads, head_dim)")
    nq = q[0].shape[0]
    if outs is None:
        outs = [torch.empty(nq, head_dim, dtype=torch.float32, device=x.device) for x in q]
    scale = 1.0 / math.sqrt(head_dim) if scale is None else float(scale)
    kr, kp, kn, kdt = _exact_arrays(k_exact, k_exact_pos, d)
    vr, vp, vn, vdt = _exact_arrays(v_exact, v_exact_pos, d)
    edt = kdt if any(kn) else vdt
    if any(kn) and any(vn) and kdt != vdt:
        raise ValueError("exact keys and values must share a dtype")
    need = lib.iskv_attention_workspace_size(n, d, max(k_hists[0].r_max, v_hists[0].r_max),
                                             k_hists[0].n_cap,
                                             max(n_total), nq)
    w = ws if ws is not None else _ws(k_hists[0].device, need)
    P = ctypes.c_void_p * n
    _lib.check(lib.iskv_decode_attention_batched(
        _handles(k_hists), _handles(v_hists), n, P(*kr), P(*kp), (ctypes.c_int64 * n)(*kn),
        P(*vr), P(*vp), (ctypes.c_int64 * n)(*vn), edt, (ctypes.c_int64 * n)(*n_total), nq,
        n_kv_heads, head_dim, float(theta), scale, P(*[x.data_ptr() for x in q]),
        P(*[o.data_ptr() for o in outs]), w.data_ptr(), w.numel(), _stream(stream)),
        "decode_attention")
    return outs


def decode_attention(k_hist, v_hist, k_exact, k_exact_pos, v_exact, v_exact_pos, n_total, q,
                     n_kv_heads, head_dim, theta=500000.0, scale=None, out=None, ws=None,
                     stream=None):
    """Single-pair form of :func:`decode_attention_batched`."""
    return decode_attention_batched([k_hist], [v_hist], [k_exact], [k_exact_pos], [v_exact],
                                    [v_exact_pos], [n_total], [q], n_kv_heads, head_dim, theta,
                                    scale, None if out is None else [out], ws, stream)[0]


def select_workspace_size(L, n_heads, block=8) -> int:
    return int(_lib.load().iskv_select_workspace_size(L, n_heads, block))


def select_prompt_blocks(keys, block=8, per_head=128, suffix_blocks=4, v_radius=32, ws=None,
                         stream=None, out=None):
    """Algorithm 1 steps 2-4 on post-RoPE prompt keys ``(L, H, hd)``. Returns device tensors
    ``P_K``, ``P_V`` (int32, length L, first ``counts[0]`` / ``counts[1]`` valid), ``head_blocks``
    (H, per_head) int32 (-1 padded) and ``counts`` (2 + H,) int64."""
    lib = _lib.load()
    _need_cuda(keys)
    if keys.dim() != 3 or not keys.is_contiguous():
        raise ValueError("keys must be a contiguous (L, H, hd) tensor")
    L, H, hd = keys.shape
    dev = keys.device
    if out is None:
        out = {"P_K": torch.empty(L, dtype=torch.int32, device=dev),
               "P_V": torch.empty(L, dtype=torch.int32, device=dev),
               "head_blocks": torch.empty(H, max(per_head, 1), dtype=torch.int32, device=dev),
               "counts": torch.zeros(2 + H, dtype=torch.int64, device=dev)}
    need = lib.iskv_select_workspace_size(L, H, block)
    w = ws if ws is not None else _ws(dev, need)
    _lib.check(lib.iskv_select_prompt_blocks(
        keys.data_ptr(), _dt(keys), L, H, hd, block, per_head, suffix_blocks, v_radius,
        out["P_K"].data_ptr(), out["P_V"].data_ptr(), out["head_blocks"].data_ptr(),
        out["counts"].data_ptr(), w.data_ptr(), w.numel(), _stream(stream)), "select_prompt_blocks")
    return out


# ------------------------------------------------------------------------------------------------
# Cache policy (Section 3.1, Section 3.2, Algorithm 1 steps 5-8, Algorithm 3 steps 1-6).

class ExactTable:
    """The exact rows of one side (K or V) of one (sequence, layer): protected rows, then the live
    rows (pending FIFO and unprotected window rows), ascending by position, in device tensors
    ``rows`` (cap_e, d) and ``pos`` (cap_e,) int32, with the host mirror the library keeps in
    ``self.t`` (an ``IskvExactTable``)."""

    def __init__(self, d: int, cap_e: int, window: int = 128, block: int = 64,
                 reorth_rows: int = 256, dtype=torch.bfloat16, device="cuda", refit_rows: int = 0):
        self.rows = torch.zeros(max(int(cap_e), 1), int(d), dtype=dtype, device=device)
        self.pos = torch.full((max(int(cap_e), 1),), -1, dtype=torch.int32, device=device)
        live_cap = int(window) + max(int(block), int(refit_rows))
        self.live = (ctypes.c_int32 * live_cap)()
        self.t = IskvExactTable(int(d), int(window), int(block), int(reorth_rows), _DT[dtype],
                                int(refit_rows), int(cap_e), _ptr(self.rows), _ptr(self.pos),
                                ctypes.cast(self.live, ctypes.POINTER(ctypes.c_int32)),
                                live_cap, 0, 0, -1, 0, 0, int(refit_rows) == 0)

    @property
    def n_exact(self) -> int:
        return int(self.t.n_prot + self.t.n_live)

    def exact(self):
        """``(rows, pos)`` views of the exact rows: the exact_rows / exact_pos of a reconstruction or
        a decode attention."""
        n = self.n_exact
        return self.rows[:n], self.pos[:n]

    def live_positions(self):
        return [self.live[i] for i in range(self.t.n_live)]


def cache_prefill(table: ExactTable, X, protected_pos, init_window: int, ws=None, stream=None):
    """Algorithm 1 steps 5-7 for one side: protected rows and the unprotected rows of the initial
    window go to ``table``; returns ``(comp_rows, comp_pos)``, the rows the prompt SVD compresses
    (device tensors, ascending positions). Synchronises the stream."""
    lib = _lib.load()
    _need_cuda(X, protected_pos)
    if X.dim() != 2 or not X.is_contiguous() or X.shape[1] != table.t.d:
        raise ValueError("X must be a contiguous (L, d) tensor")
    if protected_pos.dtype != torch.int32 or not protected_pos.is_contiguous():
        raise ValueError("protected_pos must be a contiguous int32 tensor")
    L = int(X.shape[0])
    comp = torch.empty(max(L, 1), table.t.d, dtype=X.dtype, device=X.device)
    comp_pos = torch.empty(max(L, 1), dtype=torch.int32, device=X.device)
    n_comp = ctypes.c_int64()
    need = lib.iskv_cache_prefill_workspace_size(init_window)
    w = ws if ws is not None else _ws(X.device, need)
    _lib.check(lib.iskv_cache_prefill(
        ctypes.byref(table.t), X.data_ptr(), _dt(X), L, protected_pos.data_ptr(),
        protected_pos.numel(), int(init_window), comp.data_ptr(), comp_pos.data_ptr(),
        ctypes.byref(n_comp), w.data_ptr(), w.numel(), _stream(stream)), "cache_prefill")
    return comp[:n_comp.value], comp_pos[:n_comp.value]


def compress_prompt_workspace_size(count, d, r_max, block) -> int:
    return int(_lib.load().iskv_compress_prompt_workspace_size(count, d, r_max, block))


def compress_prompt(hists, rows, positions, block: int = 64, tau_rel: float = 0.0, ws=None,
                    stream=None):
    """Algorithm 1 step 7 on the device: fold each history's compressed prompt rows
    (``rows[i]`` (n_i, d), ``positions[i]`` int32 -- what :func:`cache_prefill` returns) in blocks
    of ``block`` rows (a short last block padded with zero rows that are dropped again)."""
    if isinstance(hists, LowRankHistory):
        hists, rows, positions = [hists], [rows], [positions]
    lib = _lib.load()
    n = len(hists)
    d = hists[0].d
    rp, pp, nr = [], [], []
    dt = ISKV_F32
    for x, p in zip(rows, positions):
        if x is None or p is None or p.numel() == 0:
            rp.append(None)
            pp.append(None)
            nr.append(0)
            continue
        _need_cuda(x, p)
        if p.dtype != torch.int32 or x.shape != (p.numel(), d) or not x.is_contiguous():
            raise ValueError("rows must be (n, d) contiguous with int32 positions")
        dt = _dt(x)
        rp.append(x.data_ptr())
        pp.append(p.data_ptr())
        nr.append(p.numel())
    need = lib.iskv_compress_prompt_workspace_size(n, d, hists[0].r_max, block)
    w = ws if ws is not None else _ws(hists[0].device, need)
    P = ctypes.c_void_p * n
    _lib.check(lib.iskv_compress_prompt(_handles(hists), n, P(*rp), P(*pp),
                                        (ctypes.c_int64 * n)(*nr), dt, int(block), float(tau_rel),
                                        w.data_ptr(), w.numel(), _stream(stream)), "compress_prompt")


def cache_step_workspace_size(count, d, r_max, block, n_cap, refit_rows=0) -> int:
    return int(_lib.load().iskv_cache_step_workspace_size(count, d, r_max, block, n_cap,
                                                          refit_rows))


class CacheBatch:
    """A fixed set of (table, history) pairs stepped together: the C arrays of table and history
    pointers, the result buffers and the workspace are built once, so that a decode step costs one
    library call."""

    def __init__(self, tables, hists, ws=None):
        n = len(tables)
        if n == 0 or len(hists) != n:
            raise ValueError("one history per table")
        self.n = n
        self.tables, self.hists = list(tables), list(hists)
        self._handles = [h.handle() for h in hists]
        self._tp = (ctypes.POINTER(IskvExactTable) * n)(*[ctypes.pointer(t.t) for t in tables])
        self._hp = (ctypes.POINTER(IskvLowRank) * n)(*[ctypes.pointer(h) for h in self._handles])
        self._folded = (ctypes.c_int32 * n)()
        self._reorthed = (ctypes.c_int32 * n)()
        h0 = hists[0]
        refit = max(int(t.t.refit_rows) for t in tables)
        need = _lib.load().iskv_cache_step_workspace_size(n, h0.d, h0.r_max, tables[0].t.block,
                                                          h0.n_cap, refit)
        self.ws = ws if ws is not None else Workspace(h0.device).get(need)

    def plan(self, advance: bool = False):
        """What the next :meth:`step` will do to each table, decided on the host alone (no device
        work): ``(folded, reorthed)`` as :meth:`step` returns them. With ``advance`` the host
        mirrors move on as that step would move them (a dry run of the schedule)."""
        h0 = self.hists[0]
        _lib.check(_lib.load().iskv_cache_plan(self._tp, self.n, h0.r_max, h0.n_cap, int(advance),
                                               self._folded, self._reorthed), "cache_plan")
        return list(self._folded), [bool(x) for x in self._reorthed]

    def step(self, new_rows, tau_rel: float = 0.0, stream=None):
        """One decode step; ``new_rows`` (count, d) holds each table's row for its next position.
        Returns ``(folded, reorthed)``: per table 0, 1 (a block fold) or 2 (the first refit), and
        a bool."""
        if new_rows.dim() != 2 or new_rows.shape[0] != self.n or not new_rows.is_contiguous() \
                or not new_rows.is_cuda:
            raise ValueError("new_rows must be a contiguous (count, d) CUDA tensor")
        _lib.check(_lib.load().iskv_cache_step(
            self._tp, self._hp, self.n, new_rows.data_ptr(), _dt(new_rows), float(tau_rel),
            self._folded, self._reorthed, self.ws.data_ptr(), self.ws.numel(), _stream(stream)),
            "cache_step")
        return list(self._folded), [bool(x) for x in self._reorthed]


def cache_step(tables, hists, new_rows, tau_rel: float = 0.0, ws=None, stream=None):
    """Algorithm 3 steps 1-6 for every (table, history) pair: ``new_rows`` (count, d) holds each
    table's row for its next position. Returns ``(folded, reorthed)``: per table 0, 1 (a block
    fold) or 2 (the first refit), and a bool. For a fixed set of tables use :class:`CacheBatch`."""
    _need_cuda(new_rows)
    if ws is None:
        h0 = hists[0]
        ws = _ws(new_rows.device, _lib.load().iskv_cache_step_workspace_size(
            len(tables), h0.d, h0.r_max, tables[0].t.block, h0.n_cap,
            max(int(t.t.refit_rows) for t in tables)))
    return CacheBatch(tables, hists, ws=ws).step(new_rows, tau_rel, stream)


# ------------------------------------------------------------------------------------------------
# Instrumentation (measurement support, not part of the method).

def stage_timing(enable: bool) -> bool:
    """Turn per-stage CUDA-event timing inside the library on or off; returns the old setting."""
    return bool(_lib.load().iskv_stage_timing(1 if enable else 0))


def stage_times(reset: bool = False):
    """{stage name: (total ms, calls)} accumulated since the last reset (waits for the events)."""
    lib = _lib.load()
    n = lib.iskv_stage_count()
    ms = (ctypes.c_double * n)()
    calls = (ctypes.c_int64 * n)()
    _lib.check(lib.iskv_stage_read(ms, calls), "stage_read")
    out = {lib.iskv_stage_name(i).decode(): (ms[i], calls[i]) for i in range(n)}
    if reset:
        lib.iskv_stage_reset()
    return out


def core_stats(reset: bool = False):
    """Work counters of the core SVD (see ``iskv_core_stats``): a dict per mode ("fold",
    "reorth") with cores, sweeps, max_sweeps, pair_checks, rotations and flops."""
    buf = (ctypes.c_int64 * 12)()
    _lib.check(_lib.load().iskv_core_stats(buf, 1 if reset else 0), "core_stats")
    keys = ("cores", "sweeps", "max_sweeps", "pair_checks", "rotations", "flops")
    return {mode: {k: int(buf[6 * i + j]) for j, k in enumerate(keys)}
            for i, mode in enumerate(("fold", "reorth"))}


def launch_count() -> int:
    """Number of kernels the library has launched in this process."""
    return int(_lib.load().iskv_launch_count())


def selftest_wait_timeout(hist, limit_ns: int = 10_000_000, stream=None):
    """Run the failure-path self-test on ``hist``'s status word: a bounded wait that nothing
    satisfies gives up after ``limit_ns`` and records ISKV_ERR_TIMEOUT (no GPU fault)."""
    _lib.check(_lib.load().iskv_selftest_wait_timeout(hist.meta.data_ptr(), int(limit_ns),
                                                      _stream(stream)), "selftest_wait_timeout")

