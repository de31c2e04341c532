"""Thin Python binding over libhq.so (argument marshalling only).

Every function here has the name of the C entry point it calls and does no
arithmetic of its own: tensors are passed as device pointers, the status code
is checked, and a non-zero status raises :class:`HqError`.  PyTorch is used for
device memory and streams only.  If ``libhq.so`` is missing, importing this
module raises: there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libhq.so")

HQ_HEAD_DIM = 128
HQ_STAGE = 64
HQ_QBUF = 64
PAGE_POSITIONS = 64
PAGE_BYTES = 10304
PAGE_KCODES, PAGE_VCODES, PAGE_KSZ, PAGE_VSZ, PAGE_VLMASK = 0, 4096, 8192, 9216, 10240
STATE_T, STATE_NPACKED, STATE_NVL, STATE_NQ, STATE_KSEL, STATE_ERR = range(6)
STATE_WORDS = 8
OP_SELECT, OP_MERGE, OP_DECODE = 0, 1, 2
DEVERR_STAGING_FULL, DEVERR_CAPACITY, DEVERR_VL_CAPACITY, DEVERR_TIMEOUT, DEVERR_PAGE = 1, 2, 4, 8, 16


class HqError(RuntimeError):
    pass


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is not built: run `python -m hybrid_precision_attention_b200.build`")
_lib = ctypes.CDLL(LIB_PATH)


class HqCacheStruct(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in ("B", "Hq", "Hkv", "D", "W", "rho_bp", "cap", "vl_cap")] + [
        (n, ctypes.c_void_p)
        for n in ("pages", "kf", "vf", "vl_pos", "kr", "vr", "qbuf", "vl_sel", "state", "page_table", "score_acc",
                  "qlse")
    ] + [("n_pages", ctypes.c_int32), ("k_bits", ctypes.c_int32), ("v_bits", ctypes.c_int32), ("reserved", ctypes.c_int32)]


def page_layout(k_bits: int = 4, v_bits: int = 4) -> dict:
    """Page geometry of a code width pair (include/hq.h, HQ_PAGE_SUBPOS and friends)."""
    pr = 32 if k_bits + v_bits > 8 else 64
    sub = pr * (16 * k_bits + 16 * v_bits + 32)
    mask = (64 // pr) * sub
    return {"pr": pr, "sub": sub, "mask": mask, "bytes": (mask + 16 + 63) // 64 * 64,
            "kcodes": 0, "vcodes": pr * 16 * k_bits, "ksz": pr * 16 * (k_bits + v_bits),
            "vsz": pr * 16 * (k_bits + v_bits) + pr * 16}


_P = ctypes.c_void_p
_I = ctypes.c_int32
_S = ctypes.c_size_t
_CP = ctypes.POINTER(HqCacheStruct)

_lib.hq_abi_version.restype = _I
_lib.hq_status_str.restype = ctypes.c_char_p
_lib.hq_status_str.argtypes = [_I]
_lib.hq_last_error.restype = ctypes.c_char_p
_lib.hq_last_error.argtypes = []
_lib.hq_cache_validate.restype = _I
_lib.hq_cache_validate.argtypes = [_CP]
_lib.hq_workspace_bytes.restype = _S
_lib.hq_workspace_bytes.argtypes = [_CP, _I, _I]
_lib.hq_cache_reset.restype = _I
_lib.hq_cache_reset.argtypes = [_CP, _P]
_lib.hq_select_vlines.restype = _I
_lib.hq_select_vlines.argtypes = [_CP, _P, _I, _P, _I, _P, _P, _S, _P]
_lib.hq_pack_merge.restype = _I
_lib.hq_pack_merge.argtypes = [_CP, _P, _P, _I, _P, _S, _P]
_lib.hq_decode_attn.restype = _I
_lib.hq_decode_attn.argtypes = [_CP, _P, _P, _P, _P, ctypes.c_float, _P, _S, _P]
_lib.hq_decode_attn_noalloc.restype = _I
_lib.hq_decode_attn_noalloc.argtypes = [_CP, _P, _P, _P, _P, ctypes.c_float, _P]
_lib.hq_prefill_workspace_bytes.restype = _S
_lib.hq_prefill_workspace_bytes.argtypes = [_I, _I, _I, _I, _I, _I]
_lib.hq_prefill_attn.restype = _I
_lib.hq_prefill_attn.argtypes = [_I, _I, _I, _I, _I, _P, _P, _P, _P, _I, _I, _I, _I, ctypes.c_float, _P, _P, _S, _P]
PREFILL_E4M3, PREFILL_INT8_QK = 0, 1

_lib.hq_diag_stream_read.restype = _I
_lib.hq_diag_stream_read.argtypes = [_P, _S, _P, _I, _P]

EXPORTED = ("hq_abi_version", "hq_status_str", "hq_last_error", "hq_cache_validate", "hq_workspace_bytes", "hq_cache_reset",
            "hq_select_vlines", "hq_pack_merge", "hq_decode_attn", "hq_decode_attn_noalloc",
            "hq_prefill_workspace_bytes", "hq_prefill_attn", "hq_diag_stream_read")


def _check(st: int, what: str):
    if st != 0:
        detail = f" [{_lib.hq_last_error().decode()}]" if st == 5 else ""
        raise HqError(f"{what}: {_lib.hq_status_str(st).decode()} (status {st}){detail}")


def _ptr(t):
    if t is None:
        return None
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _need(t, dtype, shape, name):
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_cuda or not t.is_contiguous():
        raise HqError(f"{name}: expected contiguous CUDA {dtype} {tuple(shape)}, got {t.dtype} {tuple(t.shape)} on {t.device}")


def k_of(n: int, rho_bp: int) -> int:
    """ceil(rho * n) in integer basis points (same rule as the kernels)."""
    if n <= 0 or rho_bp <= 0:
        return 0
    return min(n, (n * rho_bp + 9999) // 10000)


def abi_version() -> int:
    return int(_lib.hq_abi_version())


class HybridCache:
    """Device buffers of one layer's hybrid cache (layout: include/hq.h, struct hq_cache).

    ``paged=True`` keeps the K4V4 store as a pool of ``n_pages`` pages (default:
    exactly the pages the batch can use) with a page table ``[B, Hkv, cap/64]``;
    ``page_order`` (optional, a permutation of the pool indices) fills the table,
    else page j of (b, h) is pool page (b*Hkv + h)*(cap/64) + j."""

    def __init__(self, B: int, Hq: int, Hkv: int, cap: int, W: int = 128, rho_bp: int = 500, vl_cap: int = None,
                 device="cuda", D: int = HQ_HEAD_DIM, paged: bool = False, n_pages: int = None, page_order=None,
                 running_scores: bool = False, decode_lse: bool = True, k_bits: int = 4, v_bits: int = 4):
        cap = ((cap + 127) // 128) * 128
        if vl_cap is None:
            vl_cap = max(16, ((k_of(max(cap - W, 0), rho_bp) + 15) // 16) * 16)
        self.B, self.Hq, self.Hkv, self.D, self.W, self.rho_bp, self.cap, self.vl_cap = B, Hq, Hkv, D, W, rho_bp, cap, vl_cap
        self.R = ((W + HQ_STAGE + 15) // 16) * 16   # HQ_RING_LEN(W)
        self.npg = cap // PAGE_POSITIONS
        self.k_bits, self.v_bits = k_bits, v_bits
        self.layout = page_layout(k_bits, v_bits)
        PB = self.layout["bytes"]
        dev = torch.device(device)
        z = lambda shape, dt: torch.zeros(shape, dtype=dt, device=dev)
        self.paged = paged
        if paged:
            self.n_pages = n_pages if n_pages is not None else B * Hkv * self.npg
            self.pages = z((self.n_pages, PB), torch.uint8)
            order = torch.arange(B * Hkv * self.npg, dtype=torch.int32) if page_order is None else \
                torch.as_tensor(page_order, dtype=torch.int32)
            self.page_table = order.reshape(B, Hkv, self.npg).to(dev).contiguous()
        else:
            self.n_pages = 0
            self.pages = z((B, Hkv, self.npg, PB), torch.uint8)
            self.page_table = None
        self.kf = z((B, Hkv, vl_cap, D), torch.float16)
        self.vf = z((B, Hkv, vl_cap, D), torch.float16)
        self.vl_pos = z((B, Hkv, vl_cap), torch.int32)
        self.kr = z((B, Hkv, self.R, D), torch.float16)
        self.vr = z((B, Hkv, self.R, D), torch.float16)
        self.qbuf = z((B, Hq, HQ_QBUF, D), torch.float16)
        self.vl_sel = z((B, Hkv, vl_cap), torch.int32)
        self.state_t = z((B, STATE_WORDS), torch.int32)
        self.score_acc = z((B, Hkv, cap), torch.float32) if running_scores else None
        self.qlse = torch.full((B, Hq, HQ_QBUF), float("nan"), dtype=torch.float32, device=dev) if decode_lse else None
        self.c = HqCacheStruct(B, Hq, Hkv, D, W, rho_bp, cap, vl_cap, *[t.data_ptr() for t in (
            self.pages, self.kf, self.vf, self.vl_pos, self.kr, self.vr, self.qbuf, self.vl_sel, self.state_t)],
            self.page_table.data_ptr() if paged else None,
            self.score_acc.data_ptr() if running_scores else None,
            self.qlse.data_ptr() if decode_lse else None, self.n_pages, k_bits, v_bits, 0)
        _check(_lib.hq_cache_validate(ctypes.byref(self.c)), "hq_cache_validate")
        self._ws = {}

    def slot(self, b: int) -> "CacheSlot":
        """Single-sequence view of batch row b (a B = 1 descriptor into the same buffers)."""
        return CacheSlot(self, b)

    def workspace(self, op: int, L: int = 0) -> torch.Tensor:
        n = int(_lib.hq_workspace_bytes(ctypes.byref(self.c), op, L))
        if n == 0:
            raise HqError("hq_workspace_bytes returned 0")
        w = self._ws.get(op)
        if w is None or w.numel() < n:
            w = torch.zeros(n, dtype=torch.uint8, device=self.pages.device)
            self._ws[op] = w
        return w

    def states(self) -> list:
        """Every sequence's state row as a dict."""
        rows = self.state_t.cpu().tolist()
        return [{"T": s[STATE_T], "n_packed": s[STATE_NPACKED], "n_vl": s[STATE_NVL], "n_q": s[STATE_NQ],
                 "k_sel": s[STATE_KSEL], "err": s[STATE_ERR]} for s in rows]

    def state(self, b: int = None) -> dict:
        """State row b; with b omitted, the rows must agree (a uniform batch) and
        the common row is returned, with the error bits of all rows OR-ed."""
        rows = self.states()
        if b is not None:
            return rows[b]
        out = dict(rows[0])
        err = 0
        for r in rows:
            err |= r["err"]
            for k in ("T", "n_packed", "n_vl", "n_q", "k_sel"):
                if r[k] != out[k]:
                    raise HqError(f"state rows differ ({k}): use state(b) or states() for a ragged batch")
        out["err"] = err
        return out

    def nbytes(self) -> int:
        ts = [self.pages, self.kf, self.vf, self.vl_pos, self.kr, self.vr, self.qbuf, self.vl_sel, self.state_t]
        for t in (self.page_table, self.score_acc, self.qlse):
            if t is not None:
                ts.append(t)
        return sum(t.numel() * t.element_size() for t in ts)

    def page_bytes(self) -> np.ndarray:
        """The K4V4 pages of every (b, h) in position order: uint8 [B, Hkv, cap/64, PAGE_BYTES] (host copy)."""
        pg = self.pages.cpu().numpy()
        if not self.paged:
            return pg
        tab = self.page_table.cpu().numpy().astype(np.int64)
        return pg[np.clip(tab, 0, self.n_pages - 1)]

    def packed(self) -> dict:
        """The packed store by position (host copies): codes kq/vq uint8 [B,Hkv,cap,16*bits],
        scale/zero words ksz/vsz uint32 [B,Hkv,cap,D/32], VL bitmap vl_bits bool [B,Hkv,cap]."""
        pg = self.page_bytes()
        B, H, npg, _ = pg.shape
        ly = self.layout
        pr, nsub = ly["pr"], 64 // ly["pr"]

        def take(off, width):
            parts = [pg[..., s * ly["sub"] + off:s * ly["sub"] + off + pr * width].reshape(B, H, npg, pr, width)
                     for s in range(nsub)]
            return np.concatenate(parts, axis=3).reshape(B, H, npg * 64, width)
        m = pg[..., ly["mask"]:ly["mask"] + 8].copy()
        bits = np.unpackbits(m, axis=-1, bitorder="little").reshape(B, H, npg * 64).astype(bool)
        return {"kq": take(ly["kcodes"], 16 * self.k_bits), "vq": take(ly["vcodes"], 16 * self.v_bits),
                "ksz": take(ly["ksz"], 16).copy().view(np.uint32), "vsz": take(ly["vsz"], 16).copy().view(np.uint32),
                "vl_bits": bits}


class CacheSlot:
    """One sequence of a HybridCache as a B = 1 cache: the descriptor's pointers
    are offset to batch row b (the page pool, when paged, is shared; the page
    table row is b's).  Accepted by every entry point of this module."""

    def __init__(self, parent: HybridCache, b: int):
        if not 0 <= b < parent.B:
            raise HqError(f"slot {b} outside the batch of {parent.B}")
        self.parent, self.b = parent, b
        self.B, self.Hq, self.Hkv, self.D, self.W = 1, parent.Hq, parent.Hkv, parent.D, parent.W
        self.rho_bp, self.cap, self.vl_cap, self.R = parent.rho_bp, parent.cap, parent.vl_cap, parent.R
        sl = lambda t: t[b:b + 1]
        self.kf, self.vf, self.vl_pos = sl(parent.kf), sl(parent.vf), sl(parent.vl_pos)
        self.kr, self.vr, self.qbuf, self.vl_sel = sl(parent.kr), sl(parent.vr), sl(parent.qbuf), sl(parent.vl_sel)
        self.state_t = sl(parent.state_t)
        self.pages = parent.pages if parent.paged else sl(parent.pages)
        self.page_table = sl(parent.page_table) if parent.paged else None
        self.score_acc = sl(parent.score_acc) if parent.score_acc is not None else None
        self.qlse = sl(parent.qlse) if parent.qlse is not None else None
        self.c = HqCacheStruct(1, self.Hq, self.Hkv, self.D, self.W, self.rho_bp, self.cap, self.vl_cap, *[
            t.data_ptr() for t in (self.pages, self.kf, self.vf, self.vl_pos, self.kr, self.vr, self.qbuf, self.vl_sel,
                                   self.state_t)], self.page_table.data_ptr() if parent.paged else None,
            self.score_acc.data_ptr() if self.score_acc is not None else None,
            self.qlse.data_ptr() if self.qlse is not None else None, parent.n_pages, parent.k_bits, parent.v_bits, 0)
        self.k_bits, self.v_bits, self.layout = parent.k_bits, parent.v_bits, parent.layout
        _check(_lib.hq_cache_validate(ctypes.byref(self.c)), "hq_cache_validate (slot)")
        self._ws = {}

    workspace = HybridCache.workspace

    def state(self, b: int = None) -> dict:
        return self.parent.state(self.b)


# ----------------------------------------------------------------------------- entry points

def hq_cache_reset(cache: HybridCache, stream=None):
    _check(_lib.hq_cache_reset(ctypes.byref(cache.c), _stream(stream)), "hq_cache_reset")


def hq_select_vlines(cache: HybridCache, k_dense=None, q_ext=None, scores_out=None, stream=None):
    """Init mode when k_dense [B,Hkv,L,D] and q_ext [B,Hq,nq,D] are given, else decode mode."""
    L = nq = 0
    if k_dense is not None:
        L = k_dense.shape[2]
        nq = q_ext.shape[2]
        _need(k_dense, torch.float16, (cache.B, cache.Hkv, L, cache.D), "k_dense")
        _need(q_ext, torch.float16, (cache.B, cache.Hq, nq, cache.D), "q_ext")
    if scores_out is not None:
        _need(scores_out, torch.float32, (cache.B, cache.Hkv, cache.cap), "scores_out")
    ws = cache.workspace(OP_SELECT, L)
    _check(_lib.hq_select_vlines(ctypes.byref(cache.c), _ptr(k_dense), L, _ptr(q_ext), nq, _ptr(scores_out),
                                 _ptr(ws), ws.numel(), _stream(stream)), "hq_select_vlines")


def hq_pack_merge(cache: HybridCache, k_dense=None, v_dense=None, stream=None):
    """Init mode with dense K/V [B,Hkv,L,D]; merge mode with neither."""
    L = 0
    if k_dense is not None:
        L = k_dense.shape[2]
        _need(k_dense, torch.float16, (cache.B, cache.Hkv, L, cache.D), "k_dense")
        _need(v_dense, torch.float16, (cache.B, cache.Hkv, L, cache.D), "v_dense")
    ws = cache.workspace(OP_MERGE)
    _check(_lib.hq_pack_merge(ctypes.byref(cache.c), _ptr(k_dense), _ptr(v_dense), L, _ptr(ws), ws.numel(),
                              _stream(stream)), "hq_pack_merge")


def hq_decode_attn(cache: HybridCache, q, k_new, v_new, out=None, sm_scale: float = None, stream=None):
    _need(q, torch.float16, (cache.B, cache.Hq, cache.D), "q")
    _need(k_new, torch.float16, (cache.B, cache.Hkv, cache.D), "k_new")
    _need(v_new, torch.float16, (cache.B, cache.Hkv, cache.D), "v_new")
    if out is None:
        out = torch.empty_like(q)
    _need(out, torch.float16, (cache.B, cache.Hq, cache.D), "out")
    if sm_scale is None:
        sm_scale = cache.D ** -0.5
    ws = cache.workspace(OP_DECODE)
    _check(_lib.hq_decode_attn(ctypes.byref(cache.c), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(out),
                               ctypes.c_float(sm_scale), _ptr(ws), ws.numel(), _stream(stream)), "hq_decode_attn")
    return out


def hq_decode_attn_noalloc(cache: HybridCache, q, k_new, v_new, out=None, sm_scale: float = None, stream=None):
    """hq_decode_attn for callers that may not allocate device memory: no
    workspace argument, the library's fixed scratch array is used instead (see
    include/hq.h for its size and sharing rules)."""
    _need(q, torch.float16, (cache.B, cache.Hq, cache.D), "q")
    _need(k_new, torch.float16, (cache.B, cache.Hkv, cache.D), "k_new")
    _need(v_new, torch.float16, (cache.B, cache.Hkv, cache.D), "v_new")
    if out is None:
        out = torch.empty_like(q)
    _need(out, torch.float16, (cache.B, cache.Hq, cache.D), "out")
    if sm_scale is None:
        sm_scale = cache.D ** -0.5
    _check(_lib.hq_decode_attn_noalloc(ctypes.byref(cache.c), _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(out),
                                       ctypes.c_float(sm_scale), _stream(stream)), "hq_decode_attn_noalloc")
    return out


def hq_prefill_workspace_bytes(B, Hq, Hkv, L, vl_stride, D=HQ_HEAD_DIM) -> int:
    return int(_lib.hq_prefill_workspace_bytes(B, Hq, Hkv, L, D, vl_stride))


def prefill_ws_regions(B, Hq, Hkv, L, D=HQ_HEAD_DIM) -> dict:
    """Byte offsets of the documented prefill workspace regions (include/hq.h):
    the error word, the e4m3 codes of Q and K, the fp16 values of V."""
    Lp = (L + 127) // 128 * 128
    al = lambda x: (x + 1023) // 1024 * 1024
    q8 = al(16)
    k8 = al(q8 + B * Hq * Lp * D)
    v8 = al(k8 + B * Hkv * Lp * D)
    return {"err": 0, "q8": q8, "k8": k8, "v16": v8, "Lp": Lp}


def hq_prefill_attn(q, k, v, vl_pos, n_vl: int, W: int, sm_scale: float = None, out=None, ws=None, stream=None,
                    qk_format: int = PREFILL_E4M3):
    """q [B,Hq,L,D], k/v [B,Hkv,L,D] fp16; vl_pos int32 [B,Hkv,stride] (first n_vl ascending);
    qk_format PREFILL_E4M3 (e4m3 Q, K, V) or PREFILL_INT8_QK (INT8 Q, K and FP16 V) for the quantised keys."""
    B, Hq, L, D = q.shape
    Hkv = k.shape[1]
    _need(q, torch.float16, (B, Hq, L, D), "q")
    _need(k, torch.float16, (B, Hkv, L, D), "k")
    _need(v, torch.float16, (B, Hkv, L, D), "v")
    _need(vl_pos, torch.int32, (B, Hkv, vl_pos.shape[2]), "vl_pos")
    if out is None:
        out = torch.empty_like(q)
    n = hq_prefill_workspace_bytes(B, Hq, Hkv, L, vl_pos.shape[2], D)
    if ws is None:
        ws = torch.empty(max(n, 1), dtype=torch.uint8, device=q.device)
    if sm_scale is None:
        sm_scale = D ** -0.5
    _check(_lib.hq_prefill_attn(B, Hq, Hkv, L, D, _ptr(q), _ptr(k), _ptr(v), _ptr(vl_pos), n_vl, vl_pos.shape[2], W,
                                qk_format, ctypes.c_float(sm_scale), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "hq_prefill_attn")
    return out


def hq_diag_stream_read(buf, sink, ctas_per_sm: int = 2, stream=None):
    """Read-only HBM streaming pass over a device tensor (measurement helper)."""
    _check(_lib.hq_diag_stream_read(_ptr(buf), buf.numel() * buf.element_size(), _ptr(sink), ctas_per_sm,
                                    _stream(stream)), "hq_diag_stream_read")
