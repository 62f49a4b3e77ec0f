"""B200 (sm_100a) block-sparse self-attention for video DiTs.

A thin ctypes binding over libbsa.so (declared in include/bsa.h).  Every
function here only marshals arguments: torch tensors supply device
pointers, strides and the current CUDA stream; all work runs in the
library's CUDA kernels.  There is no CPU fallback: importing works anywhere,
but every call that reaches the device needs the built library and an
sm_100 GPU, and raises otherwise.

Low-level calls mirror the C entry points one to one (`layout`, `permute`,
`pool`, `select_topk`, `sparse_attn_fwd`, `dense_attn_fwd`, `unpermute`,
`layout_stats`, `keep_count`, `query_sizes`).  `BlockSparseAttention`
strings them together for one attention layer:

    attn = BlockSparseAttention(problem)            # allocates the buffers
    out = attn(q, k, v)                             # raster [B, N, h, d] bf16
    out = attn.host_call(q_cpu, k_cpu, v_cpu)       # host tensors, copies overlapped
"""
import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libbsa.so")
MAX_PREFIX = 8

FIXED_444 = 0
DYNAMIC_888 = 1

STATUS = {0: "BSA_OK", 1: "BSA_ERR_INVALID_ARG", 2: "BSA_ERR_SHAPE", 3: "BSA_ERR_UNSUPPORTED",
          4: "BSA_ERR_WORKSPACE", 5: "BSA_ERR_CUDA", 6: "BSA_ERR_TIMEOUT",
          7: "BSA_ERR_HOST_MEMORY"}


class BSAError(RuntimeError):
    def __init__(self, status, message):
        super().__init__("%s: %s" % (STATUS.get(status, status), message))
        self.status = status


class Problem(ctypes.Structure):
    """Mirror of bsa_problem."""
    _fields_ = [("B", ctypes.c_int32), ("heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("T", ctypes.c_int32), ("H", ctypes.c_int32), ("W", ctypes.c_int32),
                ("T_valid", ctypes.c_int32), ("H_valid", ctypes.c_int32),
                ("W_valid", ctypes.c_int32), ("n_prefix_segments", ctypes.c_int32),
                ("prefix_len", ctypes.c_int32 * MAX_PREFIX), ("keep_blocks", ctypes.c_int32),
                ("block_mode", ctypes.c_int32), ("dyn_tau", ctypes.c_float),
                ("softmax_scale", ctypes.c_float)]

    @classmethod
    def make(cls, B, heads, head_dim, T, H, W, T_valid=None, H_valid=None, W_valid=None,
             prefix=(), keep_blocks=None, keep_ratio=None, block_mode=FIXED_444, dyn_tau=1.25,
             softmax_scale=None, **_ignored):
        p = cls()
        p.B, p.heads, p.head_dim = B, heads, head_dim
        p.T, p.H, p.W = T, H, W
        p.T_valid = T if T_valid is None else T_valid
        p.H_valid = H if H_valid is None else H_valid
        p.W_valid = W if W_valid is None else W_valid
        prefix = tuple(prefix)
        if len(prefix) > MAX_PREFIX:
            raise ValueError("at most %d prefix segments" % MAX_PREFIX)
        p.n_prefix_segments = len(prefix)
        for i, n in enumerate(prefix):
            p.prefix_len[i] = n
        if keep_blocks is None:
            if keep_ratio is None:
                raise ValueError("give keep_blocks or keep_ratio")
            keep_blocks = keep_count(T * H * W // 64, keep_ratio)
        p.keep_blocks = keep_blocks
        p.block_mode = block_mode
        p.dyn_tau = dyn_tau
        p.softmax_scale = ((1.0 / math.sqrt(head_dim)) if head_dim > 0 else 0.0) \
            if softmax_scale is None else softmax_scale
        return p


class Sizes(ctypes.Structure):
    """Mirror of bsa_sizes."""
    _fields_ = [("n_tokens", ctypes.c_int64), ("n_prefix_tokens", ctypes.c_int64),
                ("n_blocks", ctypes.c_int64), ("n_prefix_blocks", ctypes.c_int64),
                ("n_video_blocks", ctypes.c_int64), ("n_regions", ctypes.c_int64),
                ("list_capacity", ctypes.c_int64), ("layout_bytes", ctypes.c_size_t),
                ("perm_tensor_bytes", ctypes.c_size_t), ("raster_tensor_bytes", ctypes.c_size_t),
                ("pool_bytes", ctypes.c_size_t), ("idx_bytes", ctypes.c_size_t),
                ("cnt_bytes", ctypes.c_size_t)]


class DeviceBuffers(ctypes.Structure):
    """Mirror of bsa_device_buffers (device pointers of one whole call)."""
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("q_raster", "k_raster", "v_raster", "o_raster", "q_perm", "k_perm", "v_perm",
                 "o_perm", "layout_buf", "q_pool", "k_pool", "idx", "cnt")]


_LIB = None
_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_SIGS = {
    "bsa_keep_count": (ctypes.c_int32, [ctypes.c_int32, ctypes.c_double]),
    "bsa_query_sizes": (ctypes.c_int, [ctypes.POINTER(Problem), ctypes.POINTER(Sizes)]),
    "bsa_layout": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _I64, _I64, _I64, _P, _P]),
    "bsa_permute": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _I64, _I64, _I64, _P, _P]),
    "bsa_pool": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _P, _P, _P, _P]),
    "bsa_permute_pool": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _P, _P, _I64, _I64, _I64,
                                        _P, _P, _P, _P, _P, _P]),
    "bsa_select_topk": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _P, _P, _P]),
    "bsa_sparse_attn_fwd": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _P, _P, _P, _P, _P,
                                           _P, _P]),
    "bsa_dense_attn_fwd": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _P, _P, _P, _P, _P]),
    "bsa_unpermute": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _P, _I64, _I64, _I64, _P]),
    "bsa_layout_stats": (ctypes.c_int, [ctypes.POINTER(Problem), _P, ctypes.POINTER(_I64), _P]),
    "bsa_forward_host": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _P, _P,
                                        ctypes.POINTER(DeviceBuffers), ctypes.c_int32, _P, _P]),
    "bsa_debug_stall_pv": (ctypes.c_int, [ctypes.c_int32]),
    "bsa_take_default_status": (ctypes.c_int, [ctypes.POINTER(ctypes.c_int32), _P]),
    "bsa_pool_raster": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _P, _I64, _I64, _I64,
                                       _P, _P, _P]),
    "bsa_sparse_attn_fwd_raster": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _P, _P, _I64,
                                                  _I64, _I64, _P, _P, _P, _I64, _I64, _I64, _P,
                                                  _P]),
    "bsa_sparse_attn_fwd_lse": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _P, _P, _P, _P,
                                               _P, _P, _P, _P]),
    "bsa_query_bwd_workspace": (ctypes.c_int, [ctypes.POINTER(Problem),
                                               ctypes.POINTER(ctypes.c_size_t)]),
    "bsa_sparse_attn_bwd": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _P, _P, _P, _P, _P,
                                           _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P, _P]),
    "bsa_select_topk_gated": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _P, _P, _P, _P]),
    "bsa_window_attn_fwd_raster": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _P, _P, _I64,
                                                  _I64, _I64, _P, _P, _I64, _I64, _I64, _P, _P]),
    "bsa_forward_noalloc": (ctypes.c_int, [ctypes.POINTER(Problem), _P, _P, _P, _I64, _I64, _I64,
                                           _P, _I64, _I64, _I64, _P, _P]),
    "bsa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "bsa_last_error": (ctypes.c_char_p, []),
}


def lib():
    """The loaded libbsa.so (raises if it has not been built)."""
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libbsa.so is missing at %s: run "
                              "`python -m block_sparse_attention_47_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            fn = getattr(L, name)
            fn.restype, fn.argtypes = res, args
        _LIB = L
    return _LIB


def _check(status):
    if status != 0:
        raise BSAError(status, lib().bsa_last_error().decode())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _raster_strides(x):
    if x.dim() != 4 or x.stride(3) != 1:
        raise ValueError("raster tensors are [B, N, heads, head_dim] with head_dim contiguous")
    return x.stride(0), x.stride(1), x.stride(2)


def keep_count(n_blocks, keep_ratio):
    return int(lib().bsa_keep_count(n_blocks, keep_ratio))


def query_sizes(prob):
    s = Sizes()
    _check(lib().bsa_query_sizes(ctypes.byref(prob), ctypes.byref(s)))
    return s


def layout(prob, k_raster, layout_buf, stream=None):
    sb, sn, sh = _raster_strides(k_raster) if k_raster is not None else (0, 0, 0)
    _check(lib().bsa_layout(ctypes.byref(prob), _ptr(k_raster), sb, sn, sh, _ptr(layout_buf),
                            _stream(stream)))


def permute(prob, layout_buf, x_raster, x_perm, stream=None):
    sb, sn, sh = _raster_strides(x_raster)
    _check(lib().bsa_permute(ctypes.byref(prob), _ptr(layout_buf), _ptr(x_raster), sb, sn, sh,
                             _ptr(x_perm), _stream(stream)))


def pool(prob, layout_buf, q_perm, k_perm, q_pool, k_pool, stream=None):
    _check(lib().bsa_pool(ctypes.byref(prob), _ptr(layout_buf), _ptr(q_perm), _ptr(k_perm),
                          _ptr(q_pool), _ptr(k_pool), _stream(stream)))


def permute_pool(prob, layout_buf, q_raster, k_raster, v_raster, q_perm, k_perm, v_perm, q_pool,
                 k_pool, stream=None):
    """permute(Q), permute(K), permute(V) and pool in one pass; Q, K and V
    must share their strides."""
    sb, sn, sh = _raster_strides(q_raster)
    if _raster_strides(k_raster) != (sb, sn, sh) or _raster_strides(v_raster) != (sb, sn, sh):
        raise ValueError("permute_pool: q, k and v must share their strides")
    _check(lib().bsa_permute_pool(ctypes.byref(prob), _ptr(layout_buf), _ptr(q_raster),
                                  _ptr(k_raster), _ptr(v_raster), sb, sn, sh, _ptr(q_perm),
                                  _ptr(k_perm), _ptr(v_perm), _ptr(q_pool), _ptr(k_pool),
                                  _stream(stream)))


def select_topk(prob, q_pool, k_pool, idx, cnt, stream=None):
    _check(lib().bsa_select_topk(ctypes.byref(prob), _ptr(q_pool), _ptr(k_pool), _ptr(idx),
                                 _ptr(cnt), _stream(stream)))


def sparse_attn_fwd(prob, layout_buf, q_perm, k_perm, v_perm, idx, cnt, o_perm, dev_status=None,
                    stream=None):
    _check(lib().bsa_sparse_attn_fwd(ctypes.byref(prob), _ptr(layout_buf), _ptr(q_perm),
                                     _ptr(k_perm), _ptr(v_perm), _ptr(idx), _ptr(cnt),
                                     _ptr(o_perm), _ptr(dev_status), _stream(stream)))


def dense_attn_fwd(prob, layout_buf, q_perm, k_perm, v_perm, o_perm, dev_status=None,
                   stream=None):
    _check(lib().bsa_dense_attn_fwd(ctypes.byref(prob), _ptr(layout_buf), _ptr(q_perm),
                                    _ptr(k_perm), _ptr(v_perm), _ptr(o_perm), _ptr(dev_status),
                                    _stream(stream)))


def unpermute(prob, layout_buf, o_perm, o_raster, stream=None):
    sb, sn, sh = _raster_strides(o_raster)
    _check(lib().bsa_unpermute(ctypes.byref(prob), _ptr(layout_buf), _ptr(o_perm), _ptr(o_raster),
                               sb, sn, sh, _stream(stream)))


def _shared_strides(*ts):
    st = _raster_strides(ts[0])
    if any(_raster_strides(t) != st for t in ts[1:]):
        raise ValueError("these raster tensors must share their strides")
    return st


def pool_raster(prob, layout_buf, q_raster, k_raster, q_pool, k_pool, stream=None):
    """Block means straight from raster Q and K (bsa_pool_raster)."""
    sb, sn, sh = _shared_strides(q_raster, k_raster)
    _check(lib().bsa_pool_raster(ctypes.byref(prob), _ptr(layout_buf), _ptr(q_raster),
                                 _ptr(k_raster), sb, sn, sh, _ptr(q_pool), _ptr(k_pool),
                                 _stream(stream)))


def sparse_attn_fwd_raster(prob, layout_buf, q, k, v, idx, cnt, out, dev_status=None,
                           stream=None):
    """Block-sparse attention on raster tensors, no permuted copies
    (bsa_sparse_attn_fwd_raster)."""
    sb, sn, sh = _shared_strides(q, k, v)
    ob, on, oh = _raster_strides(out)
    _check(lib().bsa_sparse_attn_fwd_raster(ctypes.byref(prob), _ptr(layout_buf), _ptr(q),
                                            _ptr(k), _ptr(v), sb, sn, sh, _ptr(idx), _ptr(cnt),
                                            _ptr(out), ob, on, oh, _ptr(dev_status),
                                            _stream(stream)))


def sparse_attn_fwd_lse(prob, layout_buf, q_perm, k_perm, v_perm, idx, cnt, o_perm, lse,
                        dev_status=None, stream=None):
    """Forward that also writes each row's log-sum-exp (exp2 domain) into the
    fp32 [B, heads, N] tensor lse, for the backward."""
    _check(lib().bsa_sparse_attn_fwd_lse(ctypes.byref(prob), _ptr(layout_buf), _ptr(q_perm),
                                         _ptr(k_perm), _ptr(v_perm), _ptr(idx), _ptr(cnt),
                                         _ptr(o_perm), _ptr(lse), _ptr(dev_status),
                                         _stream(stream)))


def bwd_workspace_bytes(prob):
    n = ctypes.c_size_t(0)
    _check(lib().bsa_query_bwd_workspace(ctypes.byref(prob), ctypes.byref(n)))
    return int(n.value)


def sparse_attn_bwd(prob, layout_buf, q_perm, k_perm, v_perm, o_perm, do_perm, lse, idx, cnt,
                    dq_perm, dk_perm, dv_perm, workspace, dev_status=None, stream=None):
    """Gradients dQ, dK, dV (block order) over the forward's kept tiles."""
    _check(lib().bsa_sparse_attn_bwd(ctypes.byref(prob), _ptr(layout_buf), _ptr(q_perm),
                                     _ptr(k_perm), _ptr(v_perm), _ptr(o_perm), _ptr(do_perm),
                                     _ptr(lse), _ptr(idx), _ptr(cnt), _ptr(dq_perm), _ptr(dk_perm),
                                     _ptr(dv_perm), _ptr(workspace),
                                     workspace.numel() * workspace.element_size(),
                                     _ptr(dev_status), _stream(stream)))


def select_topk_gated(prob, q_pool, k_pool, gate, idx, cnt, stream=None):
    """Top-k selection with a learned-gate score (bsa_select_topk_gated): gate
    is a device fp32 [heads, head_dim, head_dim] tensor."""
    if gate.dtype != torch.float32 or tuple(gate.shape) != (prob.heads, prob.head_dim,
                                                           prob.head_dim) or \
            not gate.is_contiguous():
        raise ValueError("gate must be a contiguous float32 [heads, head_dim, head_dim] tensor")
    _check(lib().bsa_select_topk_gated(ctypes.byref(prob), _ptr(q_pool), _ptr(k_pool), _ptr(gate),
                                       _ptr(idx), _ptr(cnt), _stream(stream)))


def window_attn_fwd_raster(prob, layout_buf, q, k, v, windows, out, dev_status=None,
                           stream=None):
    """Attention of window heads on raster tensors (bsa_window_attn_fwd_raster):
    windows is a device int32 [heads, 3] tensor of (w_t, w_y, w_x), negative =
    unbounded."""
    if windows.dtype != torch.int32 or tuple(windows.shape) != (prob.heads, 3) or \
            not windows.is_contiguous():
        raise ValueError("windows must be a contiguous int32 [heads, 3] tensor")
    sb, sn, sh = _shared_strides(q, k, v)
    ob, on, oh = _raster_strides(out)
    _check(lib().bsa_window_attn_fwd_raster(ctypes.byref(prob), _ptr(layout_buf), _ptr(q), _ptr(k),
                                            _ptr(v), sb, sn, sh, _ptr(windows), _ptr(out), ob, on,
                                            oh, _ptr(dev_status), _stream(stream)))


def forward_host(prob, q_host, k_host, v_host, o_host, buffers, heads_per_group, dev_status=None,
                 stream=None):
    """The whole call on host tensors, transfers overlapped with the
    computation by groups of heads (bsa_forward_host)."""
    for t in (q_host, k_host, v_host, o_host):
        if t.is_cuda or not t.is_contiguous() or t.dim() != 4:
            raise ValueError("host tensors are contiguous [B, N, heads, head_dim] CPU tensors")
    _check(lib().bsa_forward_host(ctypes.byref(prob), _ptr(q_host), _ptr(k_host), _ptr(v_host),
                                  _ptr(o_host), ctypes.byref(buffers), int(heads_per_group),
                                  _ptr(dev_status), _stream(stream)))


def forward_noalloc(prob, q, k, v, out, dev_status=None, stream=None):
    """The whole call on device raster tensors with the library's static
    scratch instead of caller buffers (bsa_forward_noalloc), for callers that
    cannot allocate device memory.  q, k and v must share their strides."""
    sb, sn, sh = _raster_strides(q)
    if _raster_strides(k) != (sb, sn, sh) or _raster_strides(v) != (sb, sn, sh):
        raise ValueError("q, k and v must share their strides")
    ob, on, oh = _raster_strides(out)
    _check(lib().bsa_forward_noalloc(ctypes.byref(prob), _ptr(q), _ptr(k), _ptr(v), sb, sn, sh,
                                     _ptr(out), ob, on, oh, _ptr(dev_status), _stream(stream)))


NOALLOC_SCRATCH_BYTES = 64 << 20


def default_heads_per_group(heads, groups=32):
    """The smallest divisor of `heads` that makes at most `groups` groups."""
    for hg in range(1, heads + 1):
        if heads % hg == 0 and heads // hg <= groups:
            return hg
    return heads


def debug_stall_pv(enable):
    """Test hook: while enabled, attention launches queued by the calling
    thread issue no PV, so their bounded wait runs out and BSA_ERR_TIMEOUT
    reaches the status word."""
    _check(lib().bsa_debug_stall_pv(1 if enable else 0))


def take_default_status(stream=None):
    """Read and clear the library-owned status word that receives the
    device-side errors of calls made without a dev_status (waits for the
    stream first)."""
    v = ctypes.c_int32(0)
    _check(lib().bsa_take_default_status(ctypes.byref(v), _stream(stream)))
    return int(v.value)


def layout_stats(prob, layout_buf, stream=None):
    hist = (_I64 * 7)()
    _check(lib().bsa_layout_stats(ctypes.byref(prob), _ptr(layout_buf), hist, _stream(stream)))
    return list(hist)


class BlockSparseAttention:
    """One attention layer's worth of caller-owned device buffers plus the
    six-call sequence layout -> permute -> pool -> select -> attention ->
    unpermute.  Buffers are allocated once (torch) and reused per call."""

    def __init__(self, prob, device="cuda"):
        self.prob = prob
        self.sizes = s = query_sizes(prob)
        B, h, d, N, nb = prob.B, prob.heads, prob.head_dim, s.n_tokens, s.n_blocks
        dev = torch.device(device)
        self.layout_buf = torch.empty(s.layout_bytes, dtype=torch.uint8, device=dev)
        self.qp = torch.empty((B, h, N, d), dtype=torch.bfloat16, device=dev)
        self.kp = torch.empty_like(self.qp)
        self.vp = torch.empty_like(self.qp)
        self.op = torch.empty_like(self.qp)
        self.q_pool = torch.empty((B, h, nb, d), dtype=torch.float32, device=dev)
        self.k_pool = torch.empty_like(self.q_pool)
        self.idx = torch.empty((B, h, nb, s.list_capacity), dtype=torch.int32, device=dev)
        self.cnt = torch.empty((B, h, nb), dtype=torch.int32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)

    def plan(self, q, k, stream=None):
        """layout + permute(Q, K) + pool + select: the per-call overhead."""
        p = self.prob
        layout(p, k, self.layout_buf, stream)
        permute(p, self.layout_buf, q, self.qp, stream)
        permute(p, self.layout_buf, k, self.kp, stream)
        pool(p, self.layout_buf, self.qp, self.kp, self.q_pool, self.k_pool, stream)
        select_topk(p, self.q_pool, self.k_pool, self.idx, self.cnt, stream)

    def __call__(self, q, k, v, out=None, dense=False, stream=None):
        p = self.prob
        if out is None:
            out = torch.empty_like(q)
        layout(p, k, self.layout_buf, stream)
        if _raster_strides(q) == _raster_strides(k) == _raster_strides(v):
            permute_pool(p, self.layout_buf, q, k, v, self.qp, self.kp, self.vp, self.q_pool,
                         self.k_pool, stream)
        else:
            permute(p, self.layout_buf, q, self.qp, stream)
            permute(p, self.layout_buf, k, self.kp, stream)
            permute(p, self.layout_buf, v, self.vp, stream)
            pool(p, self.layout_buf, self.qp, self.kp, self.q_pool, self.k_pool, stream)
        select_topk(p, self.q_pool, self.k_pool, self.idx, self.cnt, stream)
        if dense:
            dense_attn_fwd(p, self.layout_buf, self.qp, self.kp, self.vp, self.op, self.status,
                           stream)
        else:
            sparse_attn_fwd(p, self.layout_buf, self.qp, self.kp, self.vp, self.idx, self.cnt,
                            self.op, self.status, stream)
        unpermute(p, self.layout_buf, self.op, out, stream)
        return out

    def raster_call(self, q, k, v, out=None, stream=None):
        """The same call without permuted copies: layout -> pool_raster ->
        select -> sparse_attn_fwd_raster (q, k, v share strides, heads
        contiguous in a token row)."""
        p = self.prob
        if out is None:
            out = torch.empty_like(q)
        layout(p, k, self.layout_buf, stream)
        pool_raster(p, self.layout_buf, q, k, self.q_pool, self.k_pool, stream)
        select_topk(p, self.q_pool, self.k_pool, self.idx, self.cnt, stream)
        sparse_attn_fwd_raster(p, self.layout_buf, q, k, v, self.idx, self.cnt, out, self.status,
                               stream)
        return out

    def device_buffers(self, raster=False):
        """bsa_device_buffers over this object's buffers (raster staging
        buffers are allocated on first use).  raster=True leaves the
        permuted buffers out (NULL): the permute-free sequence runs."""
        if not hasattr(self, "_raster"):
            shape = (self.prob.B, self.sizes.n_tokens, self.prob.heads, self.prob.head_dim)
            self._raster = [torch.empty(shape, dtype=torch.bfloat16, device=self.qp.device)
                            for _ in range(4)]
        b = DeviceBuffers()
        for name, t in zip(("q_raster", "k_raster", "v_raster", "o_raster"), self._raster):
            setattr(b, name, t.data_ptr())
        for name in ("q_perm", "k_perm", "v_perm", "o_perm"):
            setattr(b, name, None if raster else getattr(self, name[0] + "p").data_ptr())
        b.layout_buf = self.layout_buf.data_ptr()
        b.q_pool, b.k_pool = self.q_pool.data_ptr(), self.k_pool.data_ptr()
        b.idx, b.cnt = self.idx.data_ptr(), self.cnt.data_ptr()
        return b

    def host_call(self, q_host, k_host, v_host, out=None, heads_per_group=None, stream=None,
                  raster=False):
        """The call on host tensors (pinned memory lets the transfers overlap
        the computation); returns the host output.  raster=True runs the
        permute-free sequence."""
        if out is None:
            out = torch.empty(q_host.shape, dtype=q_host.dtype, pin_memory=q_host.is_pinned())
        hg = heads_per_group or default_heads_per_group(self.prob.heads)
        forward_host(self.prob, q_host, k_host, v_host, out, self.device_buffers(raster), hg,
                     self.status, stream)
        return out

    def check_status(self):
        v = int(self.status.item())
        if v:
            raise BSAError(v, "device-side error reported by the attention kernel")


__all__ = ["Problem", "Sizes", "BSAError", "BlockSparseAttention", "lib", "keep_count",
           "query_sizes", "layout", "permute", "pool", "select_topk", "sparse_attn_fwd",
           "dense_attn_fwd", "unpermute", "layout_stats", "forward_host", "DeviceBuffers",
           "default_heads_per_group", "debug_stall_pv", "take_default_status",
           "forward_noalloc", "NOALLOC_SCRATCH_BYTES", "pool_raster", "sparse_attn_fwd_raster",
           "window_attn_fwd_raster", "select_topk_gated", "sparse_attn_fwd_lse",
           "bwd_workspace_bytes", "sparse_attn_bwd",
           "FIXED_444", "DYNAMIC_888", "LIB_PATH"]
