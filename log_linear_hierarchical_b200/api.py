"""Python binding of the LLSA C ABI (same names as include/llsa.h).

Torch provides device memory and streams; each call passes ``data_ptr()`` values and the
current CUDA stream to libllsa.so and raises ``LLSAError`` on a non-zero status.
"""
from __future__ import annotations

import ctypes
from dataclasses import dataclass

import torch

from . import _lib
from ._lib import LLSA_BF16, LLSA_F32, LLSAShape

_DTYPES = {torch.bfloat16: LLSA_BF16, torch.float32: LLSA_F32}


class LLSAError(RuntimeError):
    def __init__(self, fn: str, status: int):
        name = _lib.STATUS_NAMES.get(status, str(status))
        try:
            text = _lib.load().llsa_status_string(status).decode()
        except Exception:  # pragma: no cover - message only
            text = ""
        super().__init__(f"{fn} returned {name}: {text}")
        self.status = status


def make_shape(B: int, H: int, N: int, D: int, topk: int, levels: int, dtype, block: int = 16,
               log_bias: bool = False, all_top: bool = False, level1: bool = False, n_valid: int = 0,
               grid_order: bool = False, one_launch_select: bool = False, causal: bool = False) -> LLSAShape:
    """``log_bias``: the log-count enrichment variant (LLSA_FLAG_LOG_BIAS); ``all_top``: the
    all-coarsest variant (LLSA_FLAG_ALL_TOP); ``level1``: the selected blocks' level-1 pooled
    tokens join the list (LLSA_FLAG_LEVEL1).  Any combination may be set.  ``n_valid``: the
    real tokens of a padded sequence (positions from n_valid on are padding; 0 = none).
    ``grid_order``: token rows are in the row-major order of a square grid
    (LLSA_FLAG_GRID_ORDER); the path reads and writes them through its quadtree order.
    ``one_launch_select``: a step runs the pyramid and selection as one cooperative launch
    (LLSA_FLAG_ONE_LAUNCH_SELECT; same results).  ``causal``: keys at or before the query
    only (LLSA_FLAG_CAUSAL; see include/llsa.h for the reading)."""
    code = _DTYPES[dtype] if isinstance(dtype, torch.dtype) else int(dtype)
    flags = ((_lib.LLSA_FLAG_LOG_BIAS if log_bias else 0) | (_lib.LLSA_FLAG_ALL_TOP if all_top else 0)
             | (_lib.LLSA_FLAG_LEVEL1 if level1 else 0) | (_lib.LLSA_FLAG_GRID_ORDER if grid_order else 0)
             | (_lib.LLSA_FLAG_ONE_LAUNCH_SELECT if one_launch_select else 0)
             | (_lib.LLSA_FLAG_CAUSAL if causal else 0))
    return LLSAShape(B, H, N, D, block, topk, levels, code, flags, n_valid)


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise LLSAError(fn, status)


def _p(t: torch.Tensor | None, name: str = "buffer") -> int | None:
    """Device address of a contiguous CUDA tensor on the current device.  The library reads
    and writes these addresses from its kernels, so a host tensor or one on another device
    is refused here rather than faulting there."""
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError(f"{name}: LLSA buffers must be contiguous")
    if not t.is_cuda:
        raise ValueError(f"{name}: LLSA buffers must be CUDA tensors (the kernels read device memory)")
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"{name}: on {t.device}, but the current device is cuda:{torch.cuda.current_device()}")
    return t.data_ptr()


_ACT_DTYPE = {0: torch.bfloat16, 1: torch.float32}  # LLSA_BF16, LLSA_F32


def _act(shape: LLSAShape, t: torch.Tensor, name: str) -> tuple:
    """An activation (q, k, v, o, dO, dq, dk, dv, a permute's src or dst): the shape's dtype
    and exactly B*H*N*D elements.  Returns (t, name) for _ptrs."""
    want = _ACT_DTYPE.get(shape.dtype)
    if t.dtype != want:
        raise ValueError(f"{name}: dtype {t.dtype}, but the shape is {want}")
    n = shape.B * shape.H * shape.N * shape.D
    if t.numel() != n:
        raise ValueError(f"{name}: {t.numel()} elements, but the shape needs B*H*N*D = {n}")
    return t, name


def _buf(t: torch.Tensor, dtype: torch.dtype, need: int, name: str) -> tuple:
    """An internal buffer (pyramid, indices, CSR, LSE): its dtype and at least ``need`` elements."""
    if t.dtype != dtype:
        raise ValueError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.numel() < need:
        raise ValueError(f"{name}: {t.numel()} elements, the shape needs {need}")
    return t, name


def _ptrs(*checked) -> list:
    """Device addresses of (tensor, name) pairs whose dtype and size were checked: every
    argument's shape is checked before any one's residency."""
    return [_p(t, name) for t, name in checked]


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _ref(shape: LLSAShape):
    return ctypes.byref(shape)


# ----------------------------------------------------------------------------- sizes

def llsa_validate_shape(shape: LLSAShape) -> int:
    return _lib.load().llsa_validate_shape(_ref(shape))


def llsa_pyramid_elems(shape: LLSAShape) -> int:
    return _lib.load().llsa_pyramid_elems(_ref(shape))


def llsa_index_elems(shape: LLSAShape) -> int:
    return _lib.load().llsa_index_elems(_ref(shape))


def llsa_row_ptr_elems(shape: LLSAShape) -> int:
    return _lib.load().llsa_row_ptr_elems(_ref(shape))


def llsa_transpose_workspace_bytes(shape: LLSAShape) -> int:
    return _lib.load().llsa_transpose_workspace_bytes(_ref(shape))


def llsa_backward_workspace_bytes(shape: LLSAShape) -> int:
    return _lib.load().llsa_backward_workspace_bytes(_ref(shape))


# ----------------------------------------------------------------------------- the five calls

def _pyr(shape, t, name):
    return _buf(t, torch.float32, llsa_pyramid_elems(shape), name)


def _idx(shape, t, name):
    return _buf(t, torch.int32, llsa_index_elems(shape), name)


def _rp(shape, t, name):
    return _buf(t, torch.int32, llsa_row_ptr_elems(shape), name)


def _lse(shape, t, name="lse"):
    return _buf(t, torch.float32, shape.B * shape.H * shape.N, name)


def llsa_build_pyramid(shape, q, k, v, q_pyr, k_pyr, v_pyr, stream=None) -> None:
    args = _ptrs(_act(shape, q, "q"), _act(shape, k, "k"), _act(shape, v, "v"), _pyr(shape, q_pyr, "q_pyr"),
            _pyr(shape, k_pyr, "k_pyr"), _pyr(shape, v_pyr, "v_pyr"))
    _check("llsa_build_pyramid", _lib.load().llsa_build_pyramid(_ref(shape), *args, _stream(stream)))


def llsa_select(shape, q_pyr, k_pyr, idx, stream=None) -> None:
    args = _ptrs(_pyr(shape, q_pyr, "q_pyr"), _pyr(shape, k_pyr, "k_pyr"), _idx(shape, idx, "idx"))
    _check("llsa_select", _lib.load().llsa_select(_ref(shape), *args, _stream(stream)))


def llsa_index_transpose(shape, idx, row_ptr, col, workspace, stream=None) -> None:
    nbytes = workspace.numel() * workspace.element_size()
    args = _ptrs(_idx(shape, idx, "idx"), _rp(shape, row_ptr, "row_ptr"), _idx(shape, col, "col"),
            (workspace, "workspace"))
    _check("llsa_index_transpose", _lib.load().llsa_index_transpose(_ref(shape), *args, nbytes, _stream(stream)))


def llsa_index_transpose_noalloc(shape, idx, row_ptr, col, stream=None) -> None:
    """llsa_index_transpose without a workspace, for callers that cannot allocate device
    memory: the library's own fixed 8 MiB scratch array is used (calls on overlapping
    streams race on it; the first call on a device must precede any stream capture)."""
    args = _ptrs(_idx(shape, idx, "idx"), _rp(shape, row_ptr, "row_ptr"), _idx(shape, col, "col"))
    _check("llsa_index_transpose_noalloc", _lib.load().llsa_index_transpose_noalloc(_ref(shape), *args,
                                                                                  _stream(stream)))


def llsa_forward(shape, q, k, v, k_pyr, v_pyr, idx, o, lse, stream=None) -> None:
    args = _ptrs(_act(shape, q, "q"), _act(shape, k, "k"), _act(shape, v, "v"), _pyr(shape, k_pyr, "k_pyr"),
            _pyr(shape, v_pyr, "v_pyr"), _idx(shape, idx, "idx"), _act(shape, o, "o"), _lse(shape, lse))
    _check("llsa_forward", _lib.load().llsa_forward(_ref(shape), *args, _stream(stream)))


def llsa_backward(shape, q, k, v, o, lse, do, k_pyr, v_pyr, idx, row_ptr, col, dq, dk, dv, workspace,
                  stream=None) -> None:
    nbytes = workspace.numel() * workspace.element_size()
    args = _ptrs(_act(shape, q, "q"), _act(shape, k, "k"), _act(shape, v, "v"), _act(shape, o, "o"), _lse(shape, lse),
            _act(shape, do, "do"), _pyr(shape, k_pyr, "k_pyr"), _pyr(shape, v_pyr, "v_pyr"), _idx(shape, idx, "idx"),
            _rp(shape, row_ptr, "row_ptr"), _idx(shape, col, "col"), _act(shape, dq, "dq"), _act(shape, dk, "dk"),
            _act(shape, dv, "dv"), (workspace, "workspace"))
    _check("llsa_backward", _lib.load().llsa_backward(_ref(shape), *args, nbytes, _stream(stream)))


def llsa_token_permute(shape, src, dst, to_z_order: bool = True, stream=None) -> None:
    """Quadtree (Z) token order of a square token grid: row-major -> Z (``to_z_order``) or
    back; src and dst are distinct [B, H, N, D] tensors."""
    args = _ptrs(_act(shape, src, "src"), _act(shape, dst, "dst"))
    _check("llsa_token_permute", _lib.load().llsa_token_permute(_ref(shape), *args, int(bool(to_z_order)),
                                                                _stream(stream)))


def llsa_device_status(stream=None) -> int:
    code = ctypes.c_int32(0)
    _check("llsa_device_status", _lib.load().llsa_device_status(ctypes.byref(code), _stream(stream)))
    return int(code.value)


def llsa_check_bounded_wait(limit_cycles: int, stream=None) -> None:
    """Runs the kernels' bounded wait on an mbarrier that nothing will complete, with a limit
    of ``limit_cycles``; the wait gives up and the device status becomes LLSA_ERR_TIMEOUT."""
    _check("llsa_check_bounded_wait", _lib.load().llsa_check_bounded_wait(int(limit_cycles), _stream(stream)))


def llsa_gather_probe(src: torch.Tensor, tile_rows: torch.Tensor, stages: int = 4, ctas: int = 148 * 4,
                      stream=None) -> None:
    """Only the attention kernels' tile gather: 2-D TMA copies of the 16 x 64 bf16 tiles of
    ``src`` ([rows, 64] bf16) whose first rows are ``tile_rows`` (int32)."""
    if src.dtype != torch.bfloat16 or src.dim() != 2 or src.shape[1] != 64:
        raise ValueError("src must be a [rows, 64] bf16 tensor")
    if tile_rows.dtype != torch.int32:
        raise ValueError("tile_rows must be int32")
    _check("llsa_gather_probe", _lib.load().llsa_gather_probe(_p(src, "src"), src.shape[0], _p(tile_rows, "tile_rows"),
                                                              tile_rows.numel(), stages, ctas, _stream(stream)))


def llsa_kernel_name(kernel_id: int) -> str:
    return _lib.load().llsa_kernel_name(kernel_id).decode()


class LaunchTrace:
    """Context manager over llsa_trace_begin / llsa_trace_end: every kernel the library
    launches from this thread inside the block is bracketed by two CUDA events on its stream."""

    def __init__(self, capacity: int):
        self.capacity = capacity
        self.events = [torch.cuda.Event(enable_timing=True) for _ in range(2 * capacity)]
        for e in self.events:       # creates the underlying cudaEvent_t
            e.record()
        self._handles = (ctypes.c_void_p * (2 * capacity))(*[e.cuda_event for e in self.events])
        self._ids = (ctypes.c_int32 * max(1, capacity))()
        self.used = 0

    def __enter__(self):
        _check("llsa_trace_begin", _lib.load().llsa_trace_begin(self._handles, self._ids, self.capacity))
        return self

    def __exit__(self, *exc):
        used = ctypes.c_int32(0)
        _lib.load().llsa_trace_end(ctypes.byref(used))
        self.used = int(used.value)
        return False

    def launches(self):
        """[(kernel name, milliseconds)] of every traced launch; synchronises."""
        torch.cuda.synchronize()
        return [(llsa_kernel_name(self._ids[i]), self.events[2 * i].elapsed_time(self.events[2 * i + 1]))
                for i in range(self.used)]


# ----------------------------------------------------------------------------- buffers

@dataclass
class LLSABuffers:
    """Every intermediate and output of one LLSA step for one shape, on one device."""

    shape: LLSAShape
    q_pyr: torch.Tensor
    k_pyr: torch.Tensor
    v_pyr: torch.Tensor
    idx: torch.Tensor
    row_ptr: torch.Tensor
    col: torch.Tensor
    o: torch.Tensor | None
    lse: torch.Tensor
    dq: torch.Tensor | None
    dk: torch.Tensor | None
    dv: torch.Tensor | None
    ws_transpose: torch.Tensor
    ws_backward: torch.Tensor

    @staticmethod
    def allocate(shape: LLSAShape, device, dtype: torch.dtype, with_grads: bool = True) -> "LLSABuffers":
        """Every buffer of one step; ``with_grads=False`` leaves dq, dk, dv as None (the
        autograd op allocates them when its backward runs)."""
        st = llsa_validate_shape(shape)
        if st != 0:
            raise LLSAError("llsa_validate_shape", st)
        B, H, N, D = shape.B, shape.H, shape.N, shape.D
        f32 = dict(device=device, dtype=torch.float32)
        i32 = dict(device=device, dtype=torch.int32)
        npyr = llsa_pyramid_elems(shape)

        def bytes_buf(n):
            return torch.empty((n + 3) // 4, **f32)

        return LLSABuffers(
            shape=shape,
            q_pyr=torch.empty(npyr, **f32), k_pyr=torch.empty(npyr, **f32), v_pyr=torch.empty(npyr, **f32),
            idx=torch.empty(llsa_index_elems(shape), **i32),
            row_ptr=torch.empty(llsa_row_ptr_elems(shape), **i32),
            col=torch.empty(llsa_index_elems(shape), **i32),
            o=torch.empty(B, H, N, D, device=device, dtype=dtype),
            lse=torch.empty(B, H, N, **f32),
            dq=torch.empty(B, H, N, D, device=device, dtype=dtype) if with_grads else None,
            dk=torch.empty(B, H, N, D, device=device, dtype=dtype) if with_grads else None,
            dv=torch.empty(B, H, N, D, device=device, dtype=dtype) if with_grads else None,
            ws_transpose=bytes_buf(llsa_transpose_workspace_bytes(shape)),
            ws_backward=bytes_buf(llsa_backward_workspace_bytes(shape)),
        )

    # Level views of the packed, level-major buffers.
    def level_sizes(self):
        s = self.shape
        return [s.N // 16 ** l for l in range(1, s.levels + 1)]

    def pyramid_levels(self, buf: torch.Tensor):
        s = self.shape
        out, off = [], 0
        for n in self.level_sizes():
            cnt = s.B * s.H * n * s.D
            out.append(buf[off:off + cnt].view(s.B, s.H, n, s.D))
            off += cnt
        return out

    def idx_levels(self):
        s = self.shape
        out, off = [], 0
        for n in self.level_sizes():
            cnt = s.B * s.H * n * s.topk
            out.append(self.idx[off:off + cnt].view(s.B, s.H, n, s.topk))
            off += cnt
        return out

    def csr_levels(self):
        s = self.shape
        rps, cols, ro, co = [], [], 0, 0
        for n in self.level_sizes():
            rc = s.B * s.H * (n + 1)
            cc = s.B * s.H * n * s.topk
            rps.append(self.row_ptr[ro:ro + rc].view(s.B, s.H, n + 1))
            cols.append(self.col[co:co + cc].view(s.B, s.H, n * s.topk))
            ro += rc
            co += cc
        return rps, cols


def llsa_forward_path(shape, q, k, v, buf: LLSABuffers, stream=None) -> None:
    """Pyramid, selection and attention forward (steps 1, 2, 4a)."""
    llsa_build_pyramid(shape, q, k, v, buf.q_pyr, buf.k_pyr, buf.v_pyr, stream)
    llsa_select(shape, buf.q_pyr, buf.k_pyr, buf.idx, stream)
    llsa_forward(shape, q, k, v, buf.k_pyr, buf.v_pyr, buf.idx, buf.o, buf.lse, stream)


def llsa_backward_path(shape, q, k, v, do, buf: LLSABuffers, stream=None) -> None:
    """Index transpose and attention backward (steps 5, 4b), after ``llsa_forward_path``."""
    llsa_index_transpose(shape, buf.idx, buf.row_ptr, buf.col, buf.ws_transpose, stream)
    llsa_backward(shape, q, k, v, buf.o, buf.lse, do, buf.k_pyr, buf.v_pyr, buf.idx, buf.row_ptr, buf.col,
                  buf.dq, buf.dk, buf.dv, buf.ws_backward, stream)


def step_buffers(shape, q, k, v, do, buf: LLSABuffers) -> _lib.LLSAStepBuffers:
    """The ``llsa_step_buffers`` of one step over ``buf`` (raw device addresses)."""
    p = _ptrs(
        _act(shape, q, "q"), _act(shape, k, "k"), _act(shape, v, "v"), _act(shape, do, "do"),
        _pyr(shape, buf.q_pyr, "q_pyr"), _pyr(shape, buf.k_pyr, "k_pyr"), _pyr(shape, buf.v_pyr, "v_pyr"),
        _idx(shape, buf.idx, "idx"), _rp(shape, buf.row_ptr, "row_ptr"), _idx(shape, buf.col, "col"),
        _act(shape, buf.o, "o"), _lse(shape, buf.lse), _act(shape, buf.dq, "dq"), _act(shape, buf.dk, "dk"),
        _act(shape, buf.dv, "dv"), (buf.ws_transpose, "ws_transpose"), (buf.ws_backward, "ws_backward"))
    return _lib.LLSAStepBuffers(*p[:16], buf.ws_transpose.numel() * 4, p[16], buf.ws_backward.numel() * 4)


_side_streams: dict[int, torch.cuda.Stream] = {}


def side_stream(device=None) -> torch.cuda.Stream:
    """The second stream a step forks its index transpose onto (one per device)."""
    dev = torch.cuda.current_device() if device is None else torch.device(device).index
    if dev not in _side_streams:
        _side_streams[dev] = torch.cuda.Stream(device=dev)
    return _side_streams[dev]


def llsa_train_step(shape, q, k, v, do, buf: LLSABuffers, stream=None, side=None) -> None:
    """One full LLSA training step of the attention op (forward and backward) through
    ``llsa_train_step``: the index transpose runs on ``side`` (default: this module's side
    stream for the device) concurrently with the forward and dQ."""
    sb = step_buffers(shape, q, k, v, do, buf)
    side = side_stream(q.device) if side is None else side
    _check("llsa_train_step", _lib.load().llsa_train_step(_ref(shape), ctypes.byref(sb), _stream(stream),
                                                          _stream(side)))


class LLSAPlan:
    """``repeat`` training steps on fixed buffers, captured once into a CUDA graph
    (``llsa_plan_create``) and replayed by ``launch`` (``llsa_plan_launch``).  Keeps the
    tensors it was built on alive; ``close`` releases the graph."""

    def __init__(self, shape, q, k, v, do, buf: LLSABuffers, repeat: int = 1):
        self._keep = (q, k, v, do, buf)
        sb = step_buffers(shape, q, k, v, do, buf)
        handle = ctypes.c_void_p()
        _check("llsa_plan_create", _lib.load().llsa_plan_create(_ref(shape), ctypes.byref(sb), repeat,
                                                                ctypes.byref(handle)))
        self._handle = handle
        self.repeat = repeat

    def launch(self, stream=None) -> None:
        if not self._handle:
            raise LLSAError("llsa_plan_launch", 1)
        _check("llsa_plan_launch", _lib.load().llsa_plan_launch(self._handle, _stream(stream)))

    def close(self) -> None:
        if self._handle:
            torch.cuda.synchronize()
            _lib.load().llsa_plan_destroy(self._handle)
            self._handle = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ----------------------------------------------------------------------------- autograd op

class _LLSAFunction(torch.autograd.Function):
    """The op's output O is handed to autograd through ``save_for_backward`` and is not kept
    in the buffers held on ``ctx`` (a tensor returned by forward and also stored as a ctx
    attribute would close a reference cycle output -> grad_fn -> ctx -> output, which keeps
    every buffer of the call alive until the cycle collector runs).  The gradient buffers are
    allocated only when backward runs, and the ctx buffers are dropped after it."""

    @staticmethod
    def forward(ctx, q, k, v, topk: int, levels: int, flags: dict):
        B, H, N, D = q.shape
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        shape = make_shape(B, H, N, D, topk, levels, q.dtype, **flags)
        buf = LLSABuffers.allocate(shape, q.device, q.dtype, with_grads=False)
        llsa_forward_path(shape, q, k, v, buf)
        o = buf.o
        buf.o = None
        ctx.save_for_backward(q, k, v, o)
        ctx.buf = buf
        ctx.shape = shape
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o = ctx.saved_tensors
        buf, shape = ctx.buf, ctx.shape
        ctx.buf = None
        dq, dk, dv = (torch.empty_like(q) for _ in range(3))
        do = do.contiguous()
        llsa_index_transpose(shape, buf.idx, buf.row_ptr, buf.col, buf.ws_transpose)
        llsa_backward(shape, q, k, v, o, buf.lse, do, buf.k_pyr, buf.v_pyr, buf.idx, buf.row_ptr, buf.col,
                      dq, dk, dv, buf.ws_backward)
        return dq, dk, dv, None, None, None


def llsa_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, topk: int = 8, levels: int = 1,
                   log_bias: bool = False, all_top: bool = False, level1: bool = False,
                   is_causal: bool = False) -> torch.Tensor:
    """Drop-in for ``F.scaled_dot_product_attention(q, k, v, is_causal=...)`` (no dropout) on
    [B, H, N, D] CUDA tensors (D = 64 or 128), bf16 or fp32, with LLSA's hierarchical block-sparse KV lists.
    ``log_bias``, ``all_top`` and ``level1`` select the enrichment variants (see make_shape);
    ``is_causal`` the causal reading (bf16, default enrichment)."""
    flags = dict(log_bias=log_bias, all_top=all_top, level1=level1, causal=is_causal)
    return _LLSAFunction.apply(q, k, v, topk, levels, flags)


def llsa_l1(q, k, v, block_size: int = 16, topk: int = 8, **variants):
    """One pooled level (the README recommends it for sequences shorter than 16384 tokens)."""
    if block_size != 16:
        raise ValueError("block_size must be 16")
    return llsa_attention(q, k, v, topk=topk, levels=1, **variants)


def llsa_l2(q, k, v, block_size: int = 16, topk: int = 8, **variants):
    """Two pooled levels (the README recommends it from 16384 tokens on)."""
    if block_size != 16:
        raise ValueError("block_size must be 16")
    return llsa_attention(q, k, v, topk=topk, levels=2, **variants)
