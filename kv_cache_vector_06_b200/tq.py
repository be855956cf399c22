"""Python binding of libtq (ctypes): argument marshalling only.

Every step of the path runs in the CUDA library; this module only turns torch tensors into
device pointers, checks that they live on the right device with the right dtype and layout,
allocates workspaces with torch when the caller gives none, and raises on a non-zero status.
There is no CPU fallback: if libtq.so is missing or cannot be loaded, importing this module
raises.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_double, c_float, c_int, c_int32, c_int64, c_size_t, c_void_p

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtq.so")

TQ_F32, TQ_BF16 = 0, 1
STATUS = {0: "TQ_OK", 1: "TQ_EINVAL", 2: "TQ_EUNSUPPORTED", 3: "TQ_ENOMEM", 4: "TQ_ECUDA", 5: "TQ_ETIMEOUT"}


class TqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


class Spec(ctypes.Structure):
    _fields_ = [("d", c_int32), ("mse_bits", c_int32), ("qjl_m", c_int32), ("layout", c_int32),
                ("norm_bits", c_int32)]


LAYOUT_ROWS, LAYOUT_BLOCK16 = 0, 1


class PackedC(ctypes.Structure):
    _fields_ = [("codes", c_void_p), ("signs", c_void_p), ("norm", c_void_p), ("rnorm", c_void_p),
                ("capacity", c_int64)]


class AttnDesc(ctypes.Structure):
    _fields_ = [("batch", c_int32), ("n_q_heads", c_int32), ("n_kv_heads", c_int32), ("scale", c_float),
                ("seq_lens", c_void_p), ("block_table", c_void_p), ("max_blocks", c_int32),
                ("block_size", c_int32), ("ctx_stride", c_int64), ("max_seq_len", c_int32),
                ("k", PackedC), ("v", PackedC), ("sparse_v", c_float)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m kv_cache_vector_06_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    st = c_int
    sig = {
        "tq_make_codebook": (st, [c_int32, c_int32, POINTER(c_double), POINTER(c_double), POINTER(c_double)]),
        "tq_ctx_create": (st, [POINTER(Spec), c_void_p, c_void_p, c_int32, POINTER(c_void_p)]),
        "tq_ctx_create_srht": (st, [POINTER(Spec), c_void_p, c_void_p, c_int32, POINTER(c_void_p)]),
        "tq_ctx_create_polar": (st, [POINTER(Spec), c_void_p, c_void_p, c_int32, POINTER(c_void_p)]),
        "tq_polar_codebook": (st, [c_int32, c_int32, POINTER(c_double), POINTER(c_double)]),
        "tq_ctx_destroy": (st, [c_void_p]),
        "tq_ctx_layout": (st, [c_void_p, POINTER(c_int64), POINTER(c_int64)]),
        "tq_encode_workspace_size": (st, [c_void_p, c_int64, POINTER(c_size_t)]),
        "tq_encode_kv": (st, [c_void_p, c_void_p, c_int, c_int64, c_int64, c_void_p, PackedC, c_void_p,
                              c_size_t, c_void_p]),
        "tq_scores_workspace_size": (st, [c_void_p, c_int32, POINTER(c_size_t)]),
        "tq_scores": (st, [c_void_p, c_void_p, c_int, c_int32, PackedC, c_int64, c_void_p, c_void_p,
                           c_size_t, c_void_p]),
        "tq_attend_workspace_size": (st, [c_void_p, c_void_p, POINTER(AttnDesc), POINTER(c_size_t)]),
        "tq_attend_decode": (st, [c_void_p, c_void_p, POINTER(AttnDesc), c_void_p, c_int, c_void_p,
                                  c_void_p, c_size_t, c_void_p]),
        "tq_attend_decode_noalloc": (st, [c_void_p, c_void_p, POINTER(AttnDesc), c_void_p, c_int, c_void_p,
                                          c_void_p]),
        "tq_decode_step_workspace_size": (st, [c_void_p, c_void_p, POINTER(AttnDesc), c_int64, POINTER(c_size_t)]),
        "tq_decode_step": (st, [c_void_p, c_void_p, POINTER(AttnDesc), c_void_p, c_void_p, c_int, c_int64, c_void_p,
                                c_void_p, c_int, c_void_p, c_void_p, c_size_t, c_void_p]),
        "tq_device_status": (st, [c_int32, POINTER(c_int32), c_int32]),
        "tq_debug_wait_probe": (st, [c_int32, c_int32]),
        "tq_search_workspace_size": (st, [c_void_p, c_int32, c_int64, c_int32, POINTER(c_size_t)]),
        "tq_search_topk": (st, [c_void_p, c_void_p, c_int, c_int32, PackedC, c_int64, c_int32, c_void_p,
                                c_void_p, c_void_p, c_size_t, c_void_p]),
        "tq_profile_enable": (st, [c_int32]),
        "tq_profile_reset": (st, []),
        "tq_profile_read": (st, [c_int32, ctypes.c_char_p, c_int32, POINTER(c_int64), POINTER(c_double)]),
        "tq_last_error": (c_char_p, []),
        "tq_version": (c_char_p, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()


def _check(status: int):
    if status != 0:
        raise TqError(status, LIB.tq_last_error().decode())


def version() -> str:
    return LIB.tq_version().decode()


def _stream_ptr(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return TQ_F32
    if t.dtype == torch.bfloat16:
        return TQ_BF16
    raise TypeError(f"unsupported dtype {t.dtype}: float32 or bfloat16")


def _dev(t: torch.Tensor, device: int, name: str, dtype=None, contiguous=True):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda or t.device.index != device:
        raise ValueError(f"{name} must be a CUDA tensor on device {device} (got {t.device})")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype} (got {t.dtype})")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return c_void_p(t.data_ptr())


def make_polar_codebook(level: int, bits: int):
    """PolarQuant angle codebook of one level, computed by the library on the host (fp64)."""
    L = 1 << bits
    c = (c_double * L)()
    t = (c_double * max(L - 1, 1))()
    _check(LIB.tq_polar_codebook(level, bits, c, t))
    return [c[i] for i in range(L)], [t[i] for i in range(L - 1)]


def make_codebook(d: int, bits: int):
    """Lloyd-Max codebook computed by the library on the host (fp64)."""
    L = 1 << bits
    c = (c_double * L)()
    t = (c_double * max(L - 1, 1))()
    mse = c_double()
    _check(LIB.tq_make_codebook(d, bits, c, t, ctypes.byref(mse)))
    return [c[i] for i in range(L)], [t[i] for i in range(L - 1)], mse.value


class Context:
    """Quantizer constants for one tensor role, resident on one device."""

    def __init__(self, d: int, mse_bits: int, qjl_m: int, rot_signs, qjl_matrix=None, device: int = 0,
                 layout: int = LAYOUT_ROWS, qjl_signs=None, polar: bool = False, norm_bits: int = 32):
        """qjl_matrix: the dense JL matrix [qjl_m, d] (tq_ctx_create); or qjl_signs: the sign
        vector D2 [d] of the structured matrix S = P H D2 (tq_ctx_create_srht).  polar: the
        PolarQuant first stage (tq_ctx_create_polar).  norm_bits: 32 or 16, the storage of the
        norms (tq_spec.norm_bits)."""
        rs = torch.as_tensor(rot_signs).to(torch.int8).contiguous().cpu()
        if rs.numel() != d:
            raise ValueError("rot_signs must have d entries")
        self.d, self.mse_bits, self.qjl_m, self.device, self.layout = d, mse_bits, qjl_m, device, layout
        self.srht = qjl_signs is not None
        self.norm_bits = norm_bits
        self.norm_dtype = torch.float16 if norm_bits == 16 else torch.float32
        spec = Spec(d, mse_bits, qjl_m, layout, norm_bits)
        h = c_void_p()
        if self.srht:
            d2 = torch.as_tensor(qjl_signs).to(torch.int8).contiguous().cpu()
            if d2.numel() != d:
                raise ValueError("qjl_signs must have d entries")
            _check(LIB.tq_ctx_create_srht(ctypes.byref(spec), c_void_p(rs.data_ptr()), c_void_p(d2.data_ptr()),
                                          device, ctypes.byref(h)))
        else:
            if qjl_m > 0:
                S = torch.as_tensor(qjl_matrix).to(torch.float32).contiguous().cpu()
                if tuple(S.shape) != (qjl_m, d):
                    raise ValueError(f"qjl_matrix must be [{qjl_m}, {d}]")
                sptr = c_void_p(S.data_ptr())
            else:
                sptr = c_void_p(None)
            create = LIB.tq_ctx_create_polar if polar else LIB.tq_ctx_create
            _check(create(ctypes.byref(spec), c_void_p(rs.data_ptr()), sptr, device, ctypes.byref(h)))
        self.polar = polar
        self._h = h
        cb, sb = c_int64(), c_int64()
        _check(LIB.tq_ctx_layout(h, ctypes.byref(cb), ctypes.byref(sb)))
        self.code_bytes, self.sign_bytes = cb.value, sb.value

    @property
    def handle(self):
        if self._h is None:
            raise ValueError("context is closed")
        return self._h

    def close(self):
        if getattr(self, "_h", None) is not None:
            LIB.tq_ctx_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


class Packed:
    """Caller-owned packed arrays (torch tensors on the context's device), indexed by slot."""

    def __init__(self, codes, norm, signs=None, rnorm=None):
        self.codes, self.norm, self.signs, self.rnorm = codes, norm, signs, rnorm

    @staticmethod
    def allocate(ctx: Context, capacity: int) -> "Packed":
        dev = torch.device("cuda", ctx.device)
        codes = torch.zeros(capacity, ctx.code_bytes, dtype=torch.uint8, device=dev)
        norm = torch.zeros(capacity, dtype=ctx.norm_dtype, device=dev)
        signs = rnorm = None
        if ctx.qjl_m > 0:
            signs = torch.zeros(capacity, ctx.sign_bytes, dtype=torch.uint8, device=dev)
            rnorm = torch.zeros(capacity, dtype=ctx.norm_dtype, device=dev)
        return Packed(codes, norm, signs, rnorm)

    @property
    def capacity(self) -> int:
        return self.codes.shape[0]

    def c(self, ctx: Context) -> PackedC:
        if self.codes.dim() != 2 or self.codes.shape[1] != ctx.code_bytes or self.codes.dtype != torch.uint8:
            raise ValueError(f"codes must be uint8 [capacity, {ctx.code_bytes}]")
        p = PackedC(_dev(self.codes, ctx.device, "codes", torch.uint8),
                    c_void_p(None), _dev(self.norm, ctx.device, "norm", ctx.norm_dtype),
                    c_void_p(None), self.codes.shape[0])
        if self.norm.numel() < self.capacity:
            raise ValueError("norm is shorter than codes")
        if ctx.qjl_m > 0 and self.signs is not None:
            if self.signs.shape != (self.capacity, ctx.sign_bytes) or self.signs.dtype != torch.uint8:
                raise ValueError(f"signs must be uint8 [capacity, {ctx.sign_bytes}]")
            if self.rnorm is None or self.rnorm.numel() < self.capacity:
                raise ValueError("rnorm must have capacity entries")
            p.signs = _dev(self.signs, ctx.device, "signs", torch.uint8)
            p.rnorm = _dev(self.rnorm, ctx.device, "rnorm", ctx.norm_dtype)
        return p


def _workspace(nbytes: int, device: int, ws):
    if nbytes == 0:
        return c_void_p(None), 0
    if ws is None:
        ws = torch.empty(nbytes, dtype=torch.uint8, device=torch.device("cuda", device))
    return _dev(ws, device, "ws"), ws.numel() * ws.element_size()


def encode_workspace_size(ctx: Context, n: int) -> int:
    b = c_size_t()
    _check(LIB.tq_encode_workspace_size(ctx.handle, n, ctypes.byref(b)))
    return b.value


def encode_kv(ctx: Context, x: torch.Tensor, out: Packed, slots: torch.Tensor = None, ws=None, stream=None):
    """Encode the rows of x ([n, d] or [n, ld] with a row stride) into `out` at `slots`."""
    if x.dim() != 2 or x.shape[1] < ctx.d or x.stride(1) != 1:
        raise ValueError("x must be [n, >=d] with unit column stride")
    n, ld = x.shape[0], x.stride(0)
    xp = _dev(x, ctx.device, "x", contiguous=False)
    sp = c_void_p(None)
    if slots is not None:
        sp = _dev(slots, ctx.device, "slots", torch.int64)
        if slots.numel() != n:
            raise ValueError("slots must have n entries")
    w, wb = _workspace(encode_workspace_size(ctx, n), ctx.device, ws)
    _check(LIB.tq_encode_kv(ctx.handle, xp, _dtype_code(x), n, ld, sp, out.c(ctx), w, wb, _stream_ptr(stream)))
    return out


def scores_workspace_size(ctx: Context, nq: int) -> int:
    b = c_size_t()
    _check(LIB.tq_scores_workspace_size(ctx.handle, nq, ctypes.byref(b)))
    return b.value


def scores(ctx: Context, q: torch.Tensor, keys: Packed, n: int = None, out=None, ws=None, stream=None):
    """Estimated inner products [nq, n] of queries q [nq, d] with slots 0..n-1 of `keys`."""
    if q.dim() != 2 or q.shape[1] != ctx.d:
        raise ValueError(f"q must be [nq, {ctx.d}]")
    n = keys.capacity if n is None else n
    nq = q.shape[0]
    if out is None:
        out = torch.empty(nq, n, dtype=torch.float32, device=q.device)
    if tuple(out.shape) != (nq, n):
        raise ValueError("out must be [nq, n]")
    w, wb = _workspace(scores_workspace_size(ctx, nq), ctx.device, ws)
    _check(LIB.tq_scores(ctx.handle, _dev(q, ctx.device, "q"), _dtype_code(q), nq, keys.c(ctx), n,
                         _dev(out, ctx.device, "out", torch.float32), w, wb, _stream_ptr(stream)))
    return out


def make_attn_desc(kctx: Context, vctx: Context, q_shape, kcache: Packed, vcache: Packed, seq_lens,
                   max_seq_len: int, ctx_stride: int = None, block_table=None, block_size: int = 16,
                   scale: float = 0.0, n_kv_heads: int = None, sparse_v: float = 0.0) -> AttnDesc:
    batch, hq, _ = q_shape
    if n_kv_heads is None:
        raise ValueError("n_kv_heads is required")
    desc = AttnDesc()
    desc.batch, desc.n_q_heads, desc.n_kv_heads, desc.scale = batch, hq, n_kv_heads, scale
    desc.seq_lens = _dev(seq_lens, kctx.device, "seq_lens", torch.int32)
    if seq_lens.numel() != batch:
        raise ValueError("seq_lens must have batch entries")
    if block_table is not None:
        if block_table.dim() != 2 or block_table.shape[0] != batch:
            raise ValueError("block_table must be [batch, max_blocks]")
        desc.block_table = _dev(block_table, kctx.device, "block_table", torch.int32)
        desc.max_blocks = block_table.shape[1]
        desc.block_size = block_size
        desc.ctx_stride = 0
    else:
        desc.block_table = c_void_p(None)
        desc.max_blocks = 0
        desc.block_size = block_size
        desc.ctx_stride = max_seq_len if ctx_stride is None else ctx_stride
    desc.max_seq_len = max_seq_len
    desc.k = kcache.c(kctx)
    desc.v = vcache.c(vctx)
    desc.sparse_v = sparse_v
    # the descriptor holds raw device pointers: it keeps the tensors they point into alive
    desc._keep = (seq_lens, block_table, kcache, vcache)
    return desc


def attend_workspace_size(kctx: Context, vctx: Context, desc: AttnDesc) -> int:
    b = c_size_t()
    _check(LIB.tq_attend_workspace_size(kctx.handle, vctx.handle, ctypes.byref(desc), ctypes.byref(b)))
    return b.value


def attend_decode(kctx: Context, vctx: Context, q: torch.Tensor, kcache: Packed, vcache: Packed, seq_lens,
                  max_seq_len: int, n_kv_heads: int, ctx_stride: int = None, block_table=None,
                  block_size: int = 16, scale: float = 0.0, out=None, ws=None, stream=None, desc=None):
    """One decode step: q [batch, n_q_heads, d] -> out fp32 [batch, n_q_heads, d]."""
    if q.dim() != 3 or q.shape[2] != kctx.d:
        raise ValueError(f"q must be [batch, heads, {kctx.d}]")
    if desc is None:
        desc = make_attn_desc(kctx, vctx, tuple(q.shape), kcache, vcache, seq_lens, max_seq_len, ctx_stride,
                              block_table, block_size, scale, n_kv_heads)
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    w, wb = _workspace(attend_workspace_size(kctx, vctx, desc), kctx.device, ws)
    _check(LIB.tq_attend_decode(kctx.handle, vctx.handle, ctypes.byref(desc), _dev(q, kctx.device, "q"),
                                _dtype_code(q), _dev(out, kctx.device, "out", torch.float32), w, wb,
                                _stream_ptr(stream)))
    return out


def decode_step_workspace_size(kctx: Context, vctx: Context, desc: AttnDesc, n_new: int) -> int:
    b = c_size_t()
    _check(LIB.tq_decode_step_workspace_size(kctx.handle, vctx.handle, ctypes.byref(desc), n_new, ctypes.byref(b)))
    return b.value


def decode_step(kctx: Context, vctx: Context, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor,
                new_slots: torch.Tensor, desc: AttnDesc, out=None, ws=None, stream=None):
    """tq_decode_step: append k_new / v_new ([n_new, d]) at new_slots, then attend with q
    ([batch, n_q_heads, d]); desc from make_attn_desc with seq_lens already counting the new tokens."""
    if k_new.shape != v_new.shape or k_new.dim() != 2 or k_new.shape[1] != kctx.d or k_new.dtype != v_new.dtype:
        raise ValueError(f"k_new and v_new must both be [n_new, {kctx.d}] with one dtype")
    n_new = k_new.shape[0]
    if new_slots.numel() != n_new:
        raise ValueError("new_slots must have n_new entries")
    if out is None:
        out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    w, wb = _workspace(decode_step_workspace_size(kctx, vctx, desc, n_new), kctx.device, ws)
    _check(LIB.tq_decode_step(kctx.handle, vctx.handle, ctypes.byref(desc), _dev(k_new, kctx.device, "k_new"),
                              _dev(v_new, kctx.device, "v_new"), _dtype_code(k_new), n_new,
                              _dev(new_slots, kctx.device, "new_slots", torch.int64), _dev(q, kctx.device, "q"),
                              _dtype_code(q), _dev(out, kctx.device, "out", torch.float32), w, wb, _stream_ptr(stream)))
    return out


DEVFLAG_STAGING_TIMEOUT = 1


TQ_ETIMEOUT = 5


def device_status(device: int = 0, clear: bool = False) -> int:
    """TQ_DEVFLAG_* bits raised by the library's kernels on `device` (synchronizes it).  The C call
    returns TQ_ETIMEOUT when a kernel gave up a bounded wait; the flags say so here, and
    check_device() raises for it."""
    f = c_int32()
    st = LIB.tq_device_status(device, ctypes.byref(f), 1 if clear else 0)
    if st not in (0, TQ_ETIMEOUT):
        _check(st)
    return f.value


def check_device(device: int = 0, clear: bool = False):
    """Raise TqError(TQ_ETIMEOUT) if a kernel on `device` gave up waiting since the last clear."""
    f = c_int32()
    _check(LIB.tq_device_status(device, ctypes.byref(f), 1 if clear else 0))


def debug_wait_probe(device: int, polls: int):
    """Test hook: make one bounded wait of every tensor-core attention CTA run out after `polls`
    polls (0 switches it off); see tq_debug_wait_probe."""
    _check(LIB.tq_debug_wait_probe(device, polls))


NOALLOC_SCRATCH_BYTES = 8 << 20


def attend_decode_noalloc(kctx: Context, vctx: Context, q: torch.Tensor, out: torch.Tensor, desc: AttnDesc,
                          stream=None):
    """tq_attend_decode_noalloc: decode attention whose scratch is the library's fixed 8 MiB
    device array, for callers that cannot allocate device memory.  `out` must be preallocated
    (fp32 [batch, n_q_heads, d]); `desc` comes from make_attn_desc.  Calls that overlap on the GPU
    share that array and race; order them on one stream."""
    if q.dim() != 3 or q.shape[2] != kctx.d:
        raise ValueError(f"q must be [batch, heads, {kctx.d}]")
    _check(LIB.tq_attend_decode_noalloc(kctx.handle, vctx.handle, ctypes.byref(desc), _dev(q, kctx.device, "q"),
                                        _dtype_code(q), _dev(out, kctx.device, "out", torch.float32),
                                        _stream_ptr(stream)))
    return out


def search_workspace_size(ctx: Context, nq: int, n: int, k: int) -> int:
    b = c_size_t()
    _check(LIB.tq_search_workspace_size(ctx.handle, nq, n, k, ctypes.byref(b)))
    return b.value


def search_topk(ctx: Context, q: torch.Tensor, db: Packed, k: int, n: int = None, out_scores=None,
                out_idx=None, ws=None, stream=None):
    """Top-k (scores fp32 [nq, k], indices int64 [nq, k]) of queries q [nq, d] over slots 0..n-1."""
    if q.dim() != 2 or q.shape[1] != ctx.d:
        raise ValueError(f"q must be [nq, {ctx.d}]")
    n = db.capacity if n is None else n
    nq = q.shape[0]
    if out_scores is None:
        out_scores = torch.empty(nq, k, dtype=torch.float32, device=q.device)
    if out_idx is None:
        out_idx = torch.empty(nq, k, dtype=torch.int64, device=q.device)
    w, wb = _workspace(search_workspace_size(ctx, nq, n, k), ctx.device, ws)
    _check(LIB.tq_search_topk(ctx.handle, _dev(q, ctx.device, "q"), _dtype_code(q), nq, db.c(ctx), n, k,
                              _dev(out_scores, ctx.device, "out_scores", torch.float32),
                              _dev(out_idx, ctx.device, "out_idx", torch.int64), w, wb, _stream_ptr(stream)))
    return out_scores, out_idx


def profile_enable(on: bool = True):
    _check(LIB.tq_profile_enable(1 if on else 0))


def profile_reset():
    _check(LIB.tq_profile_reset())


def profile_read() -> dict:
    """{kernel name: (launches, total device ms)} since the last reset."""
    out = {}
    i = 0
    buf = ctypes.create_string_buffer(64)
    while True:
        n, ms = c_int64(), c_double()
        if LIB.tq_profile_read(i, buf, 64, ctypes.byref(n), ctypes.byref(ms)) != 0:
            break
        out[buf.value.decode()] = (n.value, ms.value)
        i += 1
    return out
