"""ctypes binding of libparallax.so (declared in include/parallax.h).

Argument marshalling only: these functions read tensor pointers, shapes and
the current torch stream, fill the C parameter structs and call the library.
Every step of the computation runs in the library's CUDA kernels.  Importing
this module loads the library and raises if it has not been built; there is
no fallback.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libparallax.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m parallax_local_linear_b200.build`")

lib = ctypes.CDLL(LIB_PATH)

PLX_F32, PLX_BF16 = 0, 1
STATUS = {0: "PLX_OK", 1: "PLX_ERR_INVALID_ARG", 2: "PLX_ERR_UNSUPPORTED", 3: "PLX_ERR_WORKSPACE",
          4: "PLX_ERR_CUDA", 5: "PLX_ERR_DEVICE_FAULT", 6: "PLX_ERR_TIMEOUT"}
DEVERR_BAD_PAGE, DEVERR_TIMEOUT, DEVERR_BAD_LENGTH, DEVERR_SINGULAR = 1, 2, 4, 8
PAGE_SIZE = 64


class DecodeParams(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("kv_len", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32),
                ("in_dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32),
                ("scale", ctypes.c_float), ("num_ctas", ctypes.c_int32)]


class PrefillParams(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("seq_len", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("in_dtype", ctypes.c_int32),
                ("out_dtype", ctypes.c_int32), ("scale", ctypes.c_float),
                ("causal", ctypes.c_int32), ("cta_pair", ctypes.c_int32)]


class PrefillPagedParams(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("total_q", ctypes.c_int32), ("max_q_len", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("max_pages_per_seq", ctypes.c_int32), ("in_dtype", ctypes.c_int32),
                ("out_dtype", ctypes.c_int32), ("scale", ctypes.c_float),
                ("causal", ctypes.c_int32)]


_vp, _i32p = ctypes.c_void_p, ctypes.c_void_p
lib.parallax_abi_version.restype = ctypes.c_int32
lib.parallax_status_string.restype = ctypes.c_char_p
lib.parallax_status_string.argtypes = [ctypes.c_int]
lib.parallax_decode_num_ctas.restype = ctypes.c_int32
lib.parallax_decode_num_ctas.argtypes = [ctypes.POINTER(DecodeParams), ctypes.c_int32]
lib.parallax_decode_workspace_size.restype = ctypes.c_size_t
lib.parallax_decode_workspace_size.argtypes = [ctypes.POINTER(DecodeParams), ctypes.c_int32]
lib.parallax_decode.restype = ctypes.c_int
lib.parallax_decode.argtypes = [_vp, _vp, _vp, _vp, _i32p, _i32p, _vp, _vp, ctypes.c_size_t,
                                ctypes.POINTER(DecodeParams), _vp]
lib.parallax_prefill.restype = ctypes.c_int
lib.parallax_prefill.argtypes = [_vp, _vp, _vp, _vp, _vp, ctypes.POINTER(PrefillParams), _vp]
lib.parallax_prefill_paged.restype = ctypes.c_int
lib.parallax_prefill_paged.argtypes = [_vp, _vp, _vp, _vp, _i32p, _i32p, _i32p, _vp,
                                       ctypes.POINTER(PrefillPagedParams), _vp]
lib.parallax_prefill_train.restype = ctypes.c_int
lib.parallax_prefill_train.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, ctypes.POINTER(PrefillParams), _vp]
lib.parallax_prefill_backward_workspace_size.restype = ctypes.c_size_t
lib.parallax_prefill_backward_workspace_size.argtypes = [ctypes.POINTER(PrefillParams)]
lib.parallax_prefill_backward.restype = ctypes.c_int
lib.parallax_prefill_backward.argtypes = [_vp] * 13 + [ctypes.c_size_t, ctypes.POINTER(PrefillParams), _vp]
lib.parallax_decode_noalloc.restype = ctypes.c_int
lib.parallax_decode_projected.argtypes = [_vp, _vp, _vp, ctypes.c_int32, _vp, _vp, _i32p, _i32p, _vp, _vp, _vp,
                                          _vp, ctypes.c_size_t, ctypes.POINTER(DecodeParams), _vp]
lib.parallax_decode_projected.restype = ctypes.c_int
lib.parallax_decode_noalloc.argtypes = [_vp, _vp, _vp, _vp, _i32p, _i32p, _vp, ctypes.POINTER(DecodeParams), _vp]
NOALLOC_SCRATCH_BYTES = 8 << 20
lib.parallax_lla_decode_workspace_size.restype = ctypes.c_size_t
lib.parallax_lla_decode_workspace_size.argtypes = [ctypes.POINTER(DecodeParams), ctypes.c_float, ctypes.c_int32]
lib.parallax_lla_decode.restype = ctypes.c_int
lib.parallax_lla_decode.argtypes = [_vp, _vp, _vp, _i32p, _i32p, ctypes.c_float, _vp, _vp, _vp, ctypes.c_size_t,
                                    ctypes.POINTER(DecodeParams), _vp]
lib.parallax_decode_plan_create.restype = ctypes.c_int
lib.parallax_decode_plan_create.argtypes = [_vp, _vp, _vp, _vp, _i32p, _i32p, _vp, _vp, ctypes.c_size_t,
                                            ctypes.POINTER(DecodeParams), ctypes.POINTER(ctypes.c_void_p)]
lib.parallax_decode_plan_run.restype = ctypes.c_int
lib.parallax_decode_plan_run.argtypes = [_vp, _vp]
lib.parallax_decode_plan_run_io.restype = ctypes.c_int
lib.parallax_decode_plan_run_io.argtypes = [_vp, _vp, _vp, _vp, _vp]
lib.parallax_decode_plan_destroy.restype = None
lib.parallax_decode_plan_destroy.argtypes = [_vp]
lib.parallax_set_wait_limit_ns.restype = ctypes.c_int
lib.parallax_set_wait_limit_ns.argtypes = [ctypes.c_uint64, ctypes.POINTER(ctypes.c_uint64)]
lib.parallax_last_cuda_error.restype = ctypes.c_int32
lib.parallax_last_cuda_error.argtypes = []
lib.parallax_cuda_error_string.restype = ctypes.c_char_p
lib.parallax_cuda_error_string.argtypes = [ctypes.c_int32]
lib.parallax_last_device_error.restype = ctypes.c_int
lib.parallax_last_device_error.argtypes = [_vp, ctypes.POINTER(ctypes.c_int32)]

SIZE_MAX = ctypes.c_size_t(-1).value


class ParallaxError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        msg = f"{what}: {STATUS.get(status, status)}"
        if status == 4:   # PLX_ERR_CUDA: name the CUDA error behind it
            code = lib.parallax_last_cuda_error()
            if code:
                msg += f" ({lib.parallax_cuda_error_string(code).decode()}, cudaError {code})"
        super().__init__(msg)


def _dtype_code(dt):
    if dt == torch.bfloat16:
        return PLX_BF16
    if dt == torch.float32:
        return PLX_F32
    raise TypeError(f"unsupported dtype {dt}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _check_cuda(name, t, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _check_sequences(batch, seq_lens, page_table):
    """seq_lens [B] int32 and page_table [B, max_pages] int32 on the device
    (either may be None): the kernels read one entry / row per sequence."""
    if seq_lens is not None and tuple(seq_lens.shape) != (batch,):
        raise ValueError(f"seq_lens must have shape ({batch},), got {tuple(seq_lens.shape)}")
    if page_table is not None:
        if page_table.dim() != 2 or page_table.shape[0] != batch:
            raise ValueError(f"page_table must be [{batch}, max_pages], got {tuple(page_table.shape)}")
        if seq_lens is None:
            raise ValueError("a paged cache needs seq_lens")
        _check_cuda("page_table", page_table, torch.int32)
    if seq_lens is not None:
        _check_cuda("seq_lens", seq_lens, torch.int32)


def _check_cache_layout(batch, num_q_heads, head_dim, k_cache, v_cache, seq_lens, page_table, kv_len):
    """Shape checks of a decode's cache and sequence tables (host-only, so
    they run before any device check): the library reads the caches through
    these shapes, so a mismatch would read outside them."""
    if k_cache.dim() != 4 or tuple(k_cache.shape) != tuple(v_cache.shape):
        raise ValueError(f"k_cache and v_cache must be 4-D and alike, got {tuple(k_cache.shape)} "
                         f"and {tuple(v_cache.shape)}")
    if k_cache.shape[-1] != head_dim:
        raise ValueError(f"the caches' head_dim {k_cache.shape[-1]} differs from the queries' {head_dim}")
    if k_cache.shape[1] < 1 or num_q_heads % k_cache.shape[1]:
        raise ValueError(f"{num_q_heads} query heads do not split into {k_cache.shape[1]} KV heads")
    if page_table is None:
        if k_cache.shape[0] != batch:
            raise ValueError(f"a contiguous cache holds one sequence per row: {k_cache.shape[0]} != {batch}")
        # The library addresses token t of (b, kv head) as row (b * Hkv + kvh) * kv_len + t,
        # so kv_len must be the cache's own row count; seq_lens limits each sequence.
        if kv_len is not None and int(kv_len) != k_cache.shape[2]:
            raise ValueError(f"kv_len {kv_len} must equal the contiguous cache's length {k_cache.shape[2]} "
                             "(use seq_lens for shorter sequences)")
    else:
        if k_cache.shape[2] != PAGE_SIZE:
            raise ValueError(f"paged caches hold {PAGE_SIZE}-token pages: got {tuple(k_cache.shape)}")
        if page_table.dim() == 2 and kv_len is not None and int(kv_len) > page_table.shape[1] * PAGE_SIZE:
            raise ValueError(f"kv_len {kv_len} exceeds the page table's {page_table.shape[1]} pages")
    if seq_lens is not None and tuple(seq_lens.shape) != (batch,):
        raise ValueError(f"seq_lens must have shape ({batch},), got {tuple(seq_lens.shape)}")
    if page_table is not None:
        if page_table.dim() != 2 or page_table.shape[0] != batch:
            raise ValueError(f"page_table must be [{batch}, max_pages], got {tuple(page_table.shape)}")
        if seq_lens is None:
            raise ValueError("a paged cache needs seq_lens")


def _check_decode_inputs(q, rho, k_cache, v_cache, seq_lens, page_table, kv_len):
    """Every check of a decode call's inputs: shapes first, then devices and dtypes."""
    if q.dim() != 3 or tuple(rho.shape) != tuple(q.shape):
        raise ValueError(f"q and rho must be [B, Hq, d] and alike, got {tuple(q.shape)} and {tuple(rho.shape)}")
    B, Hq, d = q.shape
    _check_cache_layout(B, Hq, d, k_cache, v_cache, seq_lens, page_table, kv_len)
    _check_cuda("q", q)
    for name, t in (("rho", rho), ("k_cache", k_cache), ("v_cache", v_cache)):
        _check_cuda(name, t, q.dtype)
    _check_sequences(B, seq_lens, page_table)


def _output(out, out_dtype, shape, default_dtype, device):
    """The call's output tensor and dtype.  A caller's ``out`` must have
    ``shape`` (the kernels write every element of it) and, when
    ``out_dtype`` is given, that dtype; otherwise its own dtype is the
    output dtype.  Without ``out`` a new tensor is allocated."""
    if out is None:
        dt = out_dtype or default_dtype
        return torch.empty(tuple(shape), dtype=dt, device=device), dt
    if tuple(out.shape) != tuple(shape):
        raise ValueError(f"out must have shape {tuple(shape)}, got {tuple(out.shape)}")
    if out_dtype is not None and out.dtype != out_dtype:
        raise TypeError(f"out is {out.dtype} but out_dtype is {out_dtype}")
    _check_cuda("out", out)
    return out, out.dtype


_ws_lock = threading.Lock()
_workspaces = {}


def _workspace(device, nbytes):
    """A zero-initialised workspace per device, grown on demand.

    The counter region must start at zero; the library leaves it zero after
    every call, so the buffer is zeroed only when (re)allocated.
    """
    if nbytes == 0:
        return None
    idx = device.index if device.index is not None else torch.cuda.current_device()
    with _ws_lock:
        ws = _workspaces.get(idx)
        if ws is None or ws.numel() < nbytes:
            ws = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
            _workspaces[idx] = ws
        return ws


_lla_workspaces = {}


def _lla_workspace(device, nbytes):
    """The LLA pass's scratch per device, grown on demand.  It is kept apart
    from the decode workspace: LLA writes its records over the whole buffer,
    while a decode workspace's counter region must stay zero between calls."""
    idx = device.index if device.index is not None else torch.cuda.current_device()
    with _ws_lock:
        ws = _lla_workspaces.get(idx)
        if ws is None or ws.numel() < nbytes:
            ws = torch.empty(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
            _lla_workspaces[idx] = ws
        return ws


def decode_params(q, k_cache, *, page_table=None, kv_len=None, scale=None, out_dtype=None,
                  num_ctas=0, num_pages=None):
    B, Hq, d = q.shape
    paged = page_table is not None
    Hkv = k_cache.shape[1]
    if paged:
        if k_cache.shape[2] != PAGE_SIZE:
            raise ValueError(f"paged caches hold {PAGE_SIZE}-token pages: got {tuple(k_cache.shape)}")
        max_pages = page_table.shape[1]
        L = kv_len if kv_len is not None else max_pages * PAGE_SIZE
        n_pages = k_cache.shape[0] if num_pages is None else num_pages
    else:
        max_pages = 0
        L = k_cache.shape[2] if kv_len is None else kv_len
        n_pages = 0
    scale = (1.0 / d ** 0.5) if scale is None else float(scale)
    out_dtype = q.dtype if out_dtype is None else out_dtype
    return DecodeParams(B, Hq, Hkv, d, L, PAGE_SIZE if paged else 0, n_pages, max_pages,
                        _dtype_code(q.dtype), _dtype_code(out_dtype), scale, int(num_ctas))


def decode_workspace_size(params: DecodeParams, num_sms: int = 0) -> int:
    n = lib.parallax_decode_workspace_size(ctypes.byref(params), int(num_sms))
    if n == SIZE_MAX:
        raise ParallaxError(1, "parallax_decode_workspace_size")
    return n


def decode_num_ctas(params: DecodeParams, num_sms: int = 0) -> int:
    return lib.parallax_decode_num_ctas(ctypes.byref(params), int(num_sms))


def decode(q, rho, k_cache, v_cache, scale=None, *, seq_lens=None, page_table=None, out=None,
           out_dtype=None, num_ctas=0, kv_len=None):
    """Parallax decode: out[b, h] = vbar - Sigma_KV^T rho[b, h] over sequence b.

    q, rho: [B, Hq, d] (bfloat16 or float32, the cache's dtype).
    Contiguous cache: k_cache, v_cache [B, Hkv, L, d]; ``seq_lens`` (int32
    [B], optional) limits each sequence.  Paged cache: pools [P, Hkv, 64, d]
    with ``page_table`` (int32 [B, max_pages]) and ``seq_lens`` (required).
    Returns out [B, Hq, d] in ``out_dtype`` (default: the input dtype).
    """
    _check_decode_inputs(q, rho, k_cache, v_cache, seq_lens, page_table, kv_len)
    out, out_dtype = _output(out, out_dtype, q.shape, q.dtype, q.device)
    p = decode_params(q, k_cache, page_table=page_table, kv_len=kv_len, scale=scale,
                      out_dtype=out_dtype, num_ctas=num_ctas)
    nbytes = decode_workspace_size(p)
    ws = _workspace(q.device, nbytes)
    st = lib.parallax_decode(_ptr(q), _ptr(rho), _ptr(k_cache), _ptr(v_cache), _ptr(page_table),
                             _ptr(seq_lens), _ptr(out), _ptr(ws), 0 if ws is None else ws.numel(),
                             ctypes.byref(p), _stream_ptr(q.device))
    if st != 0:
        raise ParallaxError(st, "parallax_decode")
    return out


class DecodePlan:
    """A prepared decode over fixed buffers (parallax_decode_plan_*).

    Checks and prepares ``decode(q, rho, k_cache, v_cache, ..., out=out)``
    once; each ``run()`` is one kernel launch on the current stream that
    reads the buffers' current contents.  The plan keeps references to every
    tensor it was made from (so they stay allocated at the same address) and
    owns a zeroed workspace of its own.  Runs of one plan must not overlap on
    the GPU (they share that workspace).
    """

    def __init__(self, q, rho, k_cache, v_cache, scale=None, *, out, seq_lens=None, page_table=None, num_ctas=0,
                 kv_len=None):
        _check_decode_inputs(q, rho, k_cache, v_cache, seq_lens, page_table, kv_len)
        out, out_dtype = _output(out, None, q.shape, q.dtype, q.device)
        p = decode_params(q, k_cache, page_table=page_table, kv_len=kv_len, scale=scale, out_dtype=out_dtype,
                          num_ctas=num_ctas)
        nbytes = decode_workspace_size(p)
        ws = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=q.device)
        handle = ctypes.c_void_p()
        st = lib.parallax_decode_plan_create(_ptr(q), _ptr(rho), _ptr(k_cache), _ptr(v_cache), _ptr(page_table),
                                             _ptr(seq_lens), _ptr(out), _ptr(ws), ws.numel(), ctypes.byref(p),
                                             ctypes.byref(handle))
        if st != 0:
            raise ParallaxError(st, "parallax_decode_plan_create")
        self._handle = handle
        self._keep = (q, rho, k_cache, v_cache, seq_lens, page_table, ws)
        self.out = out
        self._device = q.device
        self._run = lib.parallax_decode_plan_run

    def run(self):
        st = self._run(self._handle, ctypes.c_void_p(torch.cuda.current_stream(self._device).cuda_stream))
        if st != 0:
            raise ParallaxError(st, "parallax_decode_plan_run")
        return self.out

    def run_io(self, host_q, host_rho, host_out):
        """One step from host memory on the current stream: ``host_q`` and
        ``host_rho`` in, the decode, the output into ``host_out`` (host
        tensors: contiguous, shaped and typed like q / out).  When all three
        are pinned the kernel reads and writes them across PCIe itself, and
        reads q and rho as it starts, possibly before the kernel queued
        ahead of it has finished: the host must have written them before
        the call.  Otherwise they go through copies into and out of the
        plan's buffers."""
        q, rho = self._keep[0], self._keep[1]
        for name, t, like in (("host_q", host_q, q), ("host_rho", host_rho, rho), ("host_out", host_out, self.out)):
            if t.is_cuda or not t.is_contiguous() or t.dtype != like.dtype or tuple(t.shape) != tuple(like.shape):
                raise ValueError(f"{name} must be a contiguous host tensor like {tuple(like.shape)} {like.dtype}")
        st = lib.parallax_decode_plan_run_io(self._handle, _ptr(host_q), _ptr(host_rho), _ptr(host_out),
                                             ctypes.c_void_p(torch.cuda.current_stream(self._device).cuda_stream))
        if st != 0:
            raise ParallaxError(st, "parallax_decode_plan_run_io")
        return host_out

    def __del__(self):
        h = getattr(self, "_handle", None)
        if h is not None and h.value:
            lib.parallax_decode_plan_destroy(h)
            self._handle = None


def decode_projected(x, w_q, w_rho, k_cache, v_cache, scale=None, *, seq_lens=None, page_table=None,
                     q_out=None, rho_out=None, out=None, out_dtype=None, num_ctas=0, kv_len=None):
    """Decode with q and rho projected from the new token's layer input in the
    same call: q[b, h] = bf16(W_Q[h] x[b]), rho[b, h] = bf16(W_R[h] x[b]),
    then ``decode``.

    x: [B, hidden] bf16; w_q, w_rho: [Hq * d, hidden] bf16 (d = the cache's
    head_dim); caches and options as in ``decode``.  Returns (out, q, rho):
    out [B, Hq, d] in ``out_dtype`` (default bf16) and the projections
    [B, Hq, d] bf16 (written into ``q_out`` / ``rho_out`` when given).
    """
    if x.dim() != 2 or w_q.dim() != 2 or w_q.shape != w_rho.shape or w_q.shape[1] != x.shape[1]:
        raise ValueError("x must be [B, hidden] and w_q, w_rho [Hq * d, hidden]")
    if k_cache.dim() != 4 or k_cache.shape != v_cache.shape:
        raise ValueError("caches must be 4-D and alike")
    d = k_cache.shape[-1]
    if w_q.shape[0] % d:
        raise ValueError("w_q rows must be a multiple of head_dim")
    B, Hq = x.shape[0], w_q.shape[0] // d
    _check_cache_layout(B, Hq, d, k_cache, v_cache, seq_lens, page_table, kv_len)
    _check_cuda("x", x, torch.bfloat16)
    for name, t in (("w_q", w_q), ("w_rho", w_rho), ("k_cache", k_cache), ("v_cache", v_cache)):
        _check_cuda(name, t, torch.bfloat16)
    if q_out is None:
        q_out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=x.device)
    if rho_out is None:
        rho_out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=x.device)
    for name, t in (("q_out", q_out), ("rho_out", rho_out)):
        _check_cuda(name, t, torch.bfloat16)
        if t.shape != (B, Hq, d):
            raise ValueError(f"{name} must be [B, Hq, d] = {(B, Hq, d)}")
    _check_sequences(B, seq_lens, page_table)
    out, out_dtype = _output(out, out_dtype, (B, Hq, d), torch.bfloat16, x.device)
    p = decode_params(q_out, k_cache, page_table=page_table, kv_len=kv_len, scale=scale,
                      out_dtype=out_dtype, num_ctas=num_ctas)
    nbytes = decode_workspace_size(p)
    ws = _workspace(x.device, nbytes)
    st = lib.parallax_decode_projected(_ptr(x), _ptr(w_q), _ptr(w_rho), int(x.shape[1]), _ptr(k_cache),
                                       _ptr(v_cache), _ptr(page_table), _ptr(seq_lens), _ptr(q_out),
                                       _ptr(rho_out), _ptr(out), _ptr(ws), 0 if ws is None else ws.numel(),
                                       ctypes.byref(p), _stream_ptr(x.device))
    if st != 0:
        raise ParallaxError(st, "parallax_decode_projected")
    return out, q_out, rho_out


def decode_noalloc(q, rho, k_cache, v_cache, scale=None, *, seq_lens=None, page_table=None, out, num_ctas=0,
                   kv_len=None):
    """Decode through parallax_decode_noalloc: no workspace, no allocation.

    For callers that cannot allocate device memory: ``out`` must be given,
    and the library's fixed device scratch (NOALLOC_SCRATCH_BYTES per GPU)
    holds the split partials.  Calls that overlap on the GPU race.
    """
    _check_decode_inputs(q, rho, k_cache, v_cache, seq_lens, page_table, kv_len)
    if out is None:
        raise ValueError("decode_noalloc needs out")
    out, out_dtype = _output(out, None, q.shape, q.dtype, q.device)
    p = decode_params(q, k_cache, page_table=page_table, kv_len=kv_len, scale=scale, out_dtype=out_dtype,
                      num_ctas=num_ctas)
    st = lib.parallax_decode_noalloc(_ptr(q), _ptr(rho), _ptr(k_cache), _ptr(v_cache), _ptr(page_table),
                                     _ptr(seq_lens), _ptr(out), ctypes.byref(p), _stream_ptr(q.device))
    if st != 0:
        raise ParallaxError(st, "parallax_decode_noalloc")
    return out


def lla_decode(q, k_cache, v_cache, scale=None, ridge=0.0, *, seq_lens=None, page_table=None, out=None,
               out_dtype=None, rho_out=None, num_ctas=0, kv_len=None):
    """Local Linear Attention with the solved probe (decode).

    Per (sequence, query head): rho* solves (S_KK + ridge I) rho* = kbar - q
    and out = vbar - S_KV^T rho*.  q: [B, Hq, 128] bf16; caches as in
    ``decode`` (bf16).  Returns (out [B, Hq, 128] in ``out_dtype``, default
    bf16; rho* [B, Hq, 128] float32, written into ``rho_out`` when given).
    """
    _check_decode_inputs(q, q, k_cache, v_cache, seq_lens, page_table, kv_len)
    if q.dtype != torch.bfloat16:
        raise TypeError("lla_decode takes bfloat16 queries and caches")
    out, out_dtype = _output(out, out_dtype, q.shape, torch.bfloat16, q.device)
    if rho_out is None:
        rho_out = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    _check_cuda("rho_out", rho_out, torch.float32)
    if tuple(rho_out.shape) != tuple(q.shape):
        raise ValueError(f"rho_out must have shape {tuple(q.shape)}")
    p = decode_params(q, k_cache, page_table=page_table, kv_len=kv_len, scale=scale, out_dtype=out_dtype,
                      num_ctas=num_ctas)
    nbytes = lib.parallax_lla_decode_workspace_size(ctypes.byref(p), float(ridge), 0)
    if nbytes == SIZE_MAX:
        raise ParallaxError(1, "parallax_lla_decode_workspace_size")
    ws = _lla_workspace(q.device, nbytes)
    st = lib.parallax_lla_decode(_ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(page_table), _ptr(seq_lens),
                                 float(ridge), _ptr(rho_out), _ptr(out), _ptr(ws), 0 if ws is None else ws.numel(),
                                 ctypes.byref(p), _stream_ptr(q.device))
    if st != 0:
        raise ParallaxError(st, "parallax_lla_decode")
    return out, rho_out


def prefill(q, rho, k, v, causal=True, scale=None, *, out=None, out_dtype=None, cta_pair=False):
    """Parallax prefill.  q, rho: [B, H, T, d] bf16; k, v: [B, Hkv, T, d] bf16.
    Row t attends to keys 0..t when causal, else to all T keys.  ``cta_pair``
    runs the two-SM kernel (tcgen05 cta_group::2) instead of one CTA per 128
    rows; the results are the same."""
    for name, t in (("q", q), ("rho", rho), ("k", k), ("v", v)):
        _check_cuda(name, t, torch.bfloat16)
    B, H, T, d = q.shape
    if rho.shape != q.shape or k.shape != v.shape or k.shape[0] != B or k.shape[2] != T or k.shape[3] != d:
        raise ValueError("shape mismatch")
    out, out_dtype = _output(out, out_dtype, q.shape, q.dtype, q.device)
    scale = (1.0 / d ** 0.5) if scale is None else float(scale)
    p = PrefillParams(B, H, k.shape[1], T, d, PLX_BF16, _dtype_code(out_dtype), scale, 1 if causal else 0,
                      1 if cta_pair else 0)
    st = lib.parallax_prefill(_ptr(q), _ptr(rho), _ptr(k), _ptr(v), _ptr(out), ctypes.byref(p),
                              _stream_ptr(q.device))
    if st != 0:
        raise ParallaxError(st, "parallax_prefill")
    return out


def _prefill_params(q, k, causal, scale, out_dtype, cta_pair=False):
    B, H, T, d = q.shape
    scale = (1.0 / d ** 0.5) if scale is None else float(scale)
    return PrefillParams(B, H, k.shape[1], T, d, PLX_BF16, _dtype_code(out_dtype), scale, 1 if causal else 0,
                         1 if cta_pair else 0)


def _check_prefill_inputs(q, rho, k, v):
    for name, t in (("q", q), ("rho", rho), ("k", k), ("v", v)):
        _check_cuda(name, t, torch.bfloat16)
    B, H, T, d = q.shape
    if rho.shape != q.shape or k.shape != v.shape or k.shape[0] != B or k.shape[2] != T or k.shape[3] != d:
        raise ValueError("shape mismatch")


def prefill_train(q, rho, k, v, causal=True, scale=None, *, out_dtype=None, cta_pair=False):
    """Prefill forward for training: returns (out, vbar, stats).

    vbar: float32 [B, H, T, d], the softmax average of the values of each
    row; stats: float32 [B, H, T, 2], (x, abar) per row with weights
    w_i = 2^(scale * log2(e) * q.k_i - x) and abar = sum_i w_i rho.k_i."""
    _check_prefill_inputs(q, rho, k, v)
    out_dtype = out_dtype or q.dtype
    out = torch.empty(q.shape, dtype=out_dtype, device=q.device)
    vbar = torch.empty(q.shape, dtype=torch.float32, device=q.device)
    stats = torch.empty(q.shape[:3] + (2,), dtype=torch.float32, device=q.device)
    p = _prefill_params(q, k, causal, scale, out_dtype, cta_pair)
    st = lib.parallax_prefill_train(_ptr(q), _ptr(rho), _ptr(k), _ptr(v), _ptr(out), _ptr(vbar), _ptr(stats),
                                    ctypes.byref(p), _stream_ptr(q.device))
    if st != 0:
        raise ParallaxError(st, "parallax_prefill_train")
    return out, vbar, stats


def prefill_backward(q, rho, k, v, out, vbar, stats, dout, causal=True, scale=None, *, grad_dtype=None):
    """Gradients (dq, drho, dk, dv) of a prefill given dout = dL/dout.

    ``out``, ``vbar``, ``stats`` come from prefill_train on the same inputs
    (out in the dtype the loss saw).  Gradients are returned in
    ``grad_dtype`` (default: out's dtype); dk, dv are summed over the query
    heads that share a KV head."""
    _check_prefill_inputs(q, rho, k, v)
    _check_cuda("dout", dout, torch.bfloat16)
    _check_cuda("out", out, out.dtype)
    _check_cuda("vbar", vbar, torch.float32)
    _check_cuda("stats", stats, torch.float32)
    rows = tuple(q.shape[:3])
    for name, t, shape in (("dout", dout, q.shape), ("out", out, q.shape), ("vbar", vbar, q.shape),
                           ("stats", stats, rows + (2,))):
        if tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    grad_dtype = grad_dtype or out.dtype
    if grad_dtype != out.dtype:
        raise ValueError("gradients are returned in out's dtype")
    p = _prefill_params(q, k, causal, scale, out.dtype)
    dq = torch.empty(q.shape, dtype=grad_dtype, device=q.device)
    drho = torch.empty(q.shape, dtype=grad_dtype, device=q.device)
    dk = torch.empty(k.shape, dtype=grad_dtype, device=q.device)
    dv = torch.empty(v.shape, dtype=grad_dtype, device=q.device)
    nbytes = lib.parallax_prefill_backward_workspace_size(ctypes.byref(p))
    ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=q.device)
    st = lib.parallax_prefill_backward(_ptr(q), _ptr(rho), _ptr(k), _ptr(v), _ptr(out), _ptr(vbar), _ptr(stats),
                                       _ptr(dout), _ptr(dq), _ptr(drho), _ptr(dk), _ptr(dv), _ptr(ws), nbytes,
                                       ctypes.byref(p), _stream_ptr(q.device))
    if st != 0:
        raise ParallaxError(st, "parallax_prefill_backward")
    return dq, drho, dk, dv


class ParallaxPrefill(torch.autograd.Function):
    """torch autograd node over prefill_train / prefill_backward (bf16 in and out)."""

    @staticmethod
    def forward(ctx, q, rho, k, v, causal=True, scale=None):
        out, vbar, stats = prefill_train(q, rho, k, v, causal, scale)
        ctx.save_for_backward(q, rho, k, v, out, vbar, stats)
        ctx.causal, ctx.scale = causal, scale
        return out

    @staticmethod
    def backward(ctx, dout):
        q, rho, k, v, out, vbar, stats = ctx.saved_tensors
        grads = prefill_backward(q, rho, k, v, out, vbar, stats, dout.to(torch.bfloat16).contiguous(),
                                 ctx.causal, ctx.scale)
        return grads + (None, None)


def prefill_paged(q, rho, k_cache, v_cache, page_table, cu_seqlens_q, seq_lens, *, max_q_len, scale=None,
                  causal=True, out=None, out_dtype=None):
    """Chunked (append) prefill over the paged cache.

    q, rho: [total_q, H, d] bf16, sequence b's queries at rows
    cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1, which are the LAST positions of
    its seq_lens[b] keys.  k_cache, v_cache: pools [P, Hkv, 64, d] bf16;
    page_table: int32 [B, max_pages]; cu_seqlens_q: int32 [B+1]; seq_lens:
    int32 [B] (all on the device).  ``max_q_len`` bounds every chunk length
    (a host int, so the call needs no device read-back).  Returns out
    [total_q, H, d]; rows outside every sequence are left as allocated.
    """
    for name, t in (("q", q), ("rho", rho), ("k_cache", k_cache), ("v_cache", v_cache)):
        _check_cuda(name, t, torch.bfloat16)
    for name, t in (("page_table", page_table), ("cu_seqlens_q", cu_seqlens_q), ("seq_lens", seq_lens)):
        _check_cuda(name, t, torch.int32)
    total_q, H, d = q.shape
    P, Hkv, ps, dk = k_cache.shape
    B = seq_lens.shape[0]
    if (rho.shape != q.shape or v_cache.shape != k_cache.shape or dk != d or page_table.dim() != 2
            or page_table.shape[0] != B or cu_seqlens_q.shape != (B + 1,)):
        raise ValueError("shape mismatch")
    out, out_dtype = _output(out, out_dtype, q.shape, q.dtype, q.device)
    scale = (1.0 / d ** 0.5) if scale is None else float(scale)
    p = PrefillPagedParams(B, H, Hkv, d, total_q, int(max_q_len), ps, P, page_table.shape[1], PLX_BF16,
                           _dtype_code(out_dtype), scale, 1 if causal else 0)
    st = lib.parallax_prefill_paged(_ptr(q), _ptr(rho), _ptr(k_cache), _ptr(v_cache), _ptr(page_table),
                                    _ptr(cu_seqlens_q), _ptr(seq_lens), _ptr(out), ctypes.byref(p),
                                    _stream_ptr(q.device))
    if st != 0:
        raise ParallaxError(st, "parallax_prefill_paged")
    return out


def last_device_error(device=None) -> int:
    """Synchronises the current stream and returns (and clears) the device error word."""
    device = device or torch.device("cuda", torch.cuda.current_device())
    code = ctypes.c_int32(0)
    st = lib.parallax_last_device_error(_stream_ptr(device), ctypes.byref(code))
    if st != 0:
        raise ParallaxError(st, "parallax_last_device_error")
    return code.value


def set_wait_limit_ns(limit_ns: int) -> int:
    """Sets the pipeline wait limit of the current device's kernels (ns) and
    returns the previous one (see parallax_set_wait_limit_ns)."""
    prev = ctypes.c_uint64(0)
    st = lib.parallax_set_wait_limit_ns(int(limit_ns), ctypes.byref(prev))
    if st != 0:
        raise ParallaxError(st, "parallax_set_wait_limit_ns")
    return prev.value
