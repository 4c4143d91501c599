"""Thin Python binding of the lora_gemm C ABI (include/lora_gemm.h).

Every function here only marshals arguments -- checks dtypes, shapes,
devices and contiguity of torch tensors, allocates outputs with torch when
the caller does not pass them, and hands raw device pointers plus the current
CUDA stream to liblora_gemm.so.  All arithmetic runs in the library's CUDA
kernels; there is no CPU path.  Importing this package fails with ImportError
when the compiled library is missing (build it with
``python lora_gemm_b200/build.py``).
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblora_gemm.so")

LG_OK = 0
LG_ERR_INVALID_ARG = 1
LG_ERR_UNSUPPORTED_SHAPE = 2
LG_ERR_MISALIGNED = 3
LG_ERR_WORKSPACE = 4
LG_ERR_CUDA = 5
LG_ERR_DEVICE_TIMEOUT = 6
LG_ERR_NOT_SM100 = 7

# Size of the built-in scratch array of lg_lora_linear_noalloc (the header's
# LG_NOALLOC_SCRATCH_BYTES).
LG_NOALLOC_SCRATCH_BYTES = 48 << 20

# Exported C symbols and their ctypes signatures (the header's declarations).
_c_void_p = ctypes.c_void_p
_SIGNATURES = {
    "lg_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "lg_version": (ctypes.c_int, []),
    "lg_launch_count": (ctypes.c_uint64, []),
    "lg_get_last_device_error": (ctypes.c_int, [_c_void_p]),
    "lg_set_wait_limit_ns": (None, [ctypes.c_uint64]),
    "lg_set_cluster_size": (ctypes.c_int, [ctypes.c_int]),
    "lg_set_kernel_variant": (ctypes.c_int, [ctypes.c_int]),
    "lg_lora_merge": (
        ctypes.c_int,
        [ctypes.c_int, ctypes.POINTER(_c_void_p), ctypes.POINTER(_c_void_p), ctypes.POINTER(ctypes.c_int),
         ctypes.POINTER(ctypes.c_float), ctypes.c_int, ctypes.c_int, _c_void_p, _c_void_p, _c_void_p],
    ),
    "lg_lora_linear_workspace_size": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int]),
    "lg_lora_linear": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
         ctypes.c_int, _c_void_p, ctypes.c_size_t, _c_void_p],
    ),
    "lg_lora_linear_mxfp8": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, ctypes.c_int64,
         ctypes.c_int, ctypes.c_int, ctypes.c_int, _c_void_p, ctypes.c_size_t, _c_void_p],
    ),
    "lg_lora_linear_swiglu_mxfp8": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p,
         ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int, _c_void_p, ctypes.c_size_t, _c_void_p],
    ),
    "lg_lora_linear_euler_workspace_size": (
        ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    ),
    "lg_lora_linear_euler": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, ctypes.c_int64, ctypes.c_int,
         ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_float, ctypes.c_float, _c_void_p, ctypes.c_size_t,
         _c_void_p],
    ),
    "lg_lora_linear_noalloc": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, _c_void_p, _c_void_p, _c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_int,
         ctypes.c_int, _c_void_p],
    ),
    "lg_mx_scale_bytes": (ctypes.c_size_t, [ctypes.c_int64, ctypes.c_int]),
    "lg_mx_quantize": (ctypes.c_int, [_c_void_p, ctypes.c_int64, ctypes.c_int, _c_void_p, _c_void_p, _c_void_p]),
    "lg_renoise": (
        ctypes.c_int,
        [_c_void_p, _c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_uint64, ctypes.c_uint64, _c_void_p],
    ),
    "lg_euler_step": (
        ctypes.c_int, [_c_void_p, _c_void_p, ctypes.c_int64, ctypes.c_float, ctypes.c_float, _c_void_p]
    ),
    "lg_shift_ladder": (
        ctypes.c_int,
        [ctypes.c_float, ctypes.c_int, ctypes.c_double, ctypes.POINTER(ctypes.c_float), ctypes.c_int,
         ctypes.POINTER(ctypes.c_int)],
    ),
    "lg_philox_u32": (ctypes.c_int, [_c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint64, _c_void_p]),
    "lg_philox_normal": (ctypes.c_int, [_c_void_p, ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint64, _c_void_p]),
}
EXPORTED_SYMBOLS = tuple(_SIGNATURES)


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"lora_gemm CUDA library not found at {LIB_PATH}; build it with `python lora_gemm_b200/build.py`"
        )
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


lib = _load()


class LoraGemmError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = lib.lg_status_string(status).decode()
        super().__init__(f"{where}: status {status} ({msg})")


def _check(status, where):
    if status != LG_OK:
        raise LoraGemmError(status, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device):
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _need(t, dtype, name, ndim=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dimensions")


def _shape(t, shape, name):
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _at_least(t, nbytes, name):
    _need(t, torch.uint8, name)
    if t.numel() < nbytes:
        raise ValueError(f"{name} holds {t.numel()} bytes, needs {nbytes}")


def _same_device(ref, *tensors):
    """Every tensor given (None skipped) on ref's device: the kernels run there."""
    for t in tensors:
        if t is not None and t.device != ref.device:
            raise ValueError(f"all tensors must be on {ref.device}, got one on {t.device}")


def _scales(pair, rows, K, what):
    codes, sc = pair
    _need(codes, torch.uint8, f"{what} codes", 2)
    _shape(codes, (rows, K), f"{what} codes")
    _at_least(sc, mx_scale_bytes(rows, K), f"{what} scales")
    return codes, sc


def status_string(status):
    return lib.lg_status_string(int(status)).decode()


def version():
    return lib.lg_version()


def launch_count():
    """Kernels launched by the library so far in this process."""
    return int(lib.lg_launch_count())


def set_wait_limit_ns(limit_ns):
    """Bound on each wait inside lora_linear's pipeline; 0 restores the default."""
    lib.lg_set_wait_limit_ns(int(limit_ns))


def set_cluster_size(g):
    """SMs sharing one token panel in lora_linear (1, 2, 4, 8; 0 = chosen per shape)."""
    _check(lib.lg_set_cluster_size(int(g)), "lg_set_cluster_size")


def set_kernel_variant(v):
    """lora_linear MMA variant: 1 single-SM, 2 SM pair, 0 chosen per shape."""
    _check(lib.lg_set_kernel_variant(int(v)), "lg_set_kernel_variant")


def get_last_device_error(device=None):
    """Synchronize the current stream and read/clear the device error word (a status code)."""
    device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    with torch.cuda.device(device):
        return lib.lg_get_last_device_error(_stream(device))


def lora_merge(As, Bs, scales, A_cat=None, B_cat=None):
    """A_cat = [s_i A_i] stacked along the rank axis, B_cat = [B_i] side by side (FP32)."""
    n = len(As)
    if n != len(Bs) or n != len(scales):
        raise ValueError("As, Bs and scales must have equal length")
    for i, (A, B) in enumerate(zip(As, Bs)):
        _need(A, torch.float32, f"A[{i}]", 2)
        _need(B, torch.float32, f"B[{i}]", 2)
    d_in = As[0].shape[1]
    d_out = Bs[0].shape[0]
    ranks = [A.shape[0] for A in As]
    for A, B in zip(As, Bs):
        if A.shape[1] != d_in or B.shape[0] != d_out or B.shape[1] != A.shape[0]:
            raise ValueError("adapter factor shapes disagree")
    R = sum(ranks)
    dev = As[0].device
    if A_cat is None:
        A_cat = torch.empty((R, d_in), dtype=torch.float32, device=dev)
    if B_cat is None:
        B_cat = torch.empty((d_out, R), dtype=torch.float32, device=dev)
    _need(A_cat, torch.float32, "A_cat", 2)
    _need(B_cat, torch.float32, "B_cat", 2)
    _shape(A_cat, (R, d_in), "A_cat")
    _shape(B_cat, (d_out, R), "B_cat")
    _same_device(A_cat, B_cat, *As, *Bs)
    a_ptrs = (ctypes.c_void_p * n)(*[A.data_ptr() for A in As])
    b_ptrs = (ctypes.c_void_p * n)(*[B.data_ptr() for B in Bs])
    r_arr = (ctypes.c_int * n)(*ranks)
    s_arr = (ctypes.c_float * n)(*[float(s) for s in scales])
    with torch.cuda.device(dev):
        st = lib.lg_lora_merge(n, a_ptrs, b_ptrs, r_arr, s_arr, d_in, d_out, _ptr(A_cat), _ptr(B_cat), _stream(dev))
    _check(st, "lg_lora_merge")
    return A_cat, B_cat


def lora_linear_workspace_size(M, K, N, R):
    return int(lib.lg_lora_linear_workspace_size(int(M), int(K), int(N), int(R)))


def lora_linear(x, W, A_cat, B_cat, y=None, workspace=None):
    """y = x W^T + (x A_cat^T) B_cat^T; bf16 x [M, K], W [N, K]; FP32 A_cat [R, K], B_cat [N, R]."""
    _need(x, torch.bfloat16, "x", 2)
    _need(W, torch.bfloat16, "W", 2)
    M, K = x.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("W must be [N, K]")
    R = 0
    if A_cat is not None and A_cat.numel() > 0:
        _need(A_cat, torch.float32, "A_cat", 2)
        _need(B_cat, torch.float32, "B_cat", 2)
        R = A_cat.shape[0]
        if A_cat.shape[1] != K or tuple(B_cat.shape) != (N, R):
            raise ValueError("A_cat must be [R, K] and B_cat [N, R]")
    else:
        A_cat = B_cat = None
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(y, torch.bfloat16, "y", 2)
    _shape(y, (M, N), "y")
    need = lora_linear_workspace_size(M, K, N, R)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _same_device(x, W, A_cat, B_cat, y, workspace)
    with torch.cuda.device(x.device):
        st = lib.lg_lora_linear(_ptr(x), _ptr(W), _ptr(A_cat), _ptr(B_cat), _ptr(y), M, K, N, R,
                                _ptr(workspace), ws_bytes, _stream(x.device))
    _check(st, "lg_lora_linear")
    return y


def mx_scale_bytes(rows, K):
    """Bytes of E8M0 scales lg_mx_quantize writes for [rows, K] (0 for an unsupported shape)."""
    return int(lib.lg_mx_scale_bytes(int(rows), int(K)))


def mx_quantize(x, codes=None, scales=None):
    """MXFP8 of bf16 rows x [rows, K] along K: (E4M3 codes uint8 [rows, K],
    E8M0 scales uint8 in the blocked layout of include/lora_gemm.h)."""
    _need(x, torch.bfloat16, "x", 2)
    rows, K = x.shape
    if codes is None:
        codes = torch.empty((rows, K), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty(max(mx_scale_bytes(rows, K), 1), dtype=torch.uint8, device=x.device)
    _need(codes, torch.uint8, "codes", 2)
    _shape(codes, (rows, K), "codes")
    _at_least(scales, mx_scale_bytes(rows, K), "scales")
    _same_device(x, codes, scales)
    with torch.cuda.device(x.device):
        st = lib.lg_mx_quantize(_ptr(x), rows, K, _ptr(codes), _ptr(scales), _stream(x.device))
    _check(st, "lg_mx_quantize")
    return codes, scales


def lora_linear_mxfp8(x, x_mx, W_mx, A_cat, B_cat, y=None, workspace=None):
    """lora_linear with the base term as MXFP8 GEMMs: x_mx = mx_quantize(x),
    W_mx = mx_quantize(W) (pairs of codes and scales); the LoRA term from the
    bf16 x.  K must be a multiple of 128."""
    _need(x, torch.bfloat16, "x", 2)
    M, K = x.shape
    _need(W_mx[0], torch.uint8, "W codes", 2)
    N = W_mx[0].shape[0]
    xq, xsf = _scales(x_mx, M, K, "x")
    wq, wsf = _scales(W_mx, N, K, "W")
    R = 0
    if A_cat is not None and A_cat.numel() > 0:
        _need(A_cat, torch.float32, "A_cat", 2)
        _need(B_cat, torch.float32, "B_cat", 2)
        R = A_cat.shape[0]
        if A_cat.shape[1] != K or tuple(B_cat.shape) != (N, R):
            raise ValueError("A_cat must be [R, K] and B_cat [N, R]")
    else:
        A_cat = B_cat = None
    if y is None:
        y = torch.empty((M, N), dtype=torch.bfloat16, device=x.device)
    _need(y, torch.bfloat16, "y", 2)
    _shape(y, (M, N), "y")
    need = lora_linear_workspace_size(M, K, N, R)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _same_device(x, xq, xsf, wq, wsf, A_cat, B_cat, y, workspace)
    with torch.cuda.device(x.device):
        st = lib.lg_lora_linear_mxfp8(_ptr(x), _ptr(xq), _ptr(xsf), _ptr(wq), _ptr(wsf), _ptr(A_cat), _ptr(B_cat),
                                      _ptr(y), M, K, N, R, _ptr(workspace), ws_bytes, _stream(x.device))
    _check(st, "lg_lora_linear_mxfp8")
    return y


def lora_linear_swiglu_mxfp8(x, x_mx, W2_mx, A_cat, B_cat, out=None, workspace=None):
    """MLP input projection with SwiGLU and the MXFP8 quantizer fused: W2 [2F, K]
    (gate rows, then up rows) as mx_quantize(W2); returns (codes [M, F], scales)
    of silu(z[:, :F]) * z[:, F:] with z = x W2^T + LoRA."""
    _need(x, torch.bfloat16, "x", 2)
    M, K = x.shape
    _need(W2_mx[0], torch.uint8, "W2 codes", 2)
    N2 = W2_mx[0].shape[0]
    if N2 % 2:
        raise ValueError("W2 must have 2F rows (gate rows, then up rows)")
    F = N2 // 2
    xq, xsf = _scales(x_mx, M, K, "x")
    wq, wsf = _scales(W2_mx, N2, K, "W2")
    R = 0
    if A_cat is not None and A_cat.numel() > 0:
        _need(A_cat, torch.float32, "A_cat", 2)
        _need(B_cat, torch.float32, "B_cat", 2)
        R = A_cat.shape[0]
        if A_cat.shape[1] != K or tuple(B_cat.shape) != (N2, R):
            raise ValueError("A_cat must be [R, K] and B_cat [2F, R]")
    else:
        A_cat = B_cat = None
    if out is None:
        out = (torch.empty((M, F), dtype=torch.uint8, device=x.device),
               torch.empty(max(mx_scale_bytes(M, F), 1), dtype=torch.uint8, device=x.device))
    _need(out[0], torch.uint8, "output codes", 2)
    _shape(out[0], (M, F), "output codes")
    _at_least(out[1], mx_scale_bytes(M, F), "output scales")
    need = lora_linear_workspace_size(M, K, N2, R)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _same_device(x, xq, xsf, wq, wsf, A_cat, B_cat, out[0], out[1], workspace)
    with torch.cuda.device(x.device):
        st = lib.lg_lora_linear_swiglu_mxfp8(_ptr(x), _ptr(xq), _ptr(xsf), _ptr(wq), _ptr(wsf), _ptr(A_cat),
                                             _ptr(B_cat), _ptr(out[0]), _ptr(out[1]), M, K, F, R, _ptr(workspace),
                                             ws_bytes, _stream(x.device))
    _check(st, "lg_lora_linear_swiglu_mxfp8")
    return out


def lora_linear_euler_workspace_size(M, K, N, R):
    return int(lib.lg_lora_linear_euler_workspace_size(int(M), int(K), int(N), int(R)))


def lora_linear_euler(x, W, A_cat, B_cat, z, sigma, sigma_next, frame_tokens, z_bf16=None, workspace=None):
    """The step's last projection with the Euler update fused: v = x W^T +
    (x A_cat^T) B_cat^T (W [C, K]) updates the FP32 latent z [frames, C,
    frame_tokens] in place, z += (sigma_next - sigma) v (token m = cell
    m mod frame_tokens of frame m // frame_tokens); z_bf16 (same shape, or
    None) receives bf16(z).  Returns z."""
    _need(x, torch.bfloat16, "x", 2)
    _need(W, torch.bfloat16, "W", 2)
    _need(z, torch.float32, "z")
    M, K = x.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("W must be [N, K]")
    if z.numel() != M * N:
        raise ValueError("z must hold M * N elements")
    if z_bf16 is not None:
        _need(z_bf16, torch.bfloat16, "z_bf16")
        if z_bf16.numel() != z.numel():
            raise ValueError("z_bf16 must have as many elements as z")
    R = 0
    if A_cat is not None and A_cat.numel() > 0:
        _need(A_cat, torch.float32, "A_cat", 2)
        _need(B_cat, torch.float32, "B_cat", 2)
        R = A_cat.shape[0]
        if A_cat.shape[1] != K or tuple(B_cat.shape) != (N, R):
            raise ValueError("A_cat must be [R, K] and B_cat [N, R]")
    else:
        A_cat = B_cat = None
    need = lora_linear_euler_workspace_size(M, K, N, R)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _same_device(x, W, A_cat, B_cat, z, z_bf16, workspace)
    with torch.cuda.device(x.device):
        st = lib.lg_lora_linear_euler(_ptr(x), _ptr(W), _ptr(A_cat), _ptr(B_cat), _ptr(z), _ptr(z_bf16), M, K, N, R,
                                      int(frame_tokens), float(sigma), float(sigma_next), _ptr(workspace), ws_bytes,
                                      _stream(x.device))
    _check(st, "lg_lora_linear_euler")
    return z


def lora_linear_noalloc(x, W, A_cat, B_cat, y):
    """lora_linear without a workspace, for callers that cannot allocate device
    memory at call time: the factor copies go to the library's built-in scratch
    array (see lg_lora_linear_noalloc in include/lora_gemm.h).  y must be given."""
    _need(x, torch.bfloat16, "x", 2)
    _need(W, torch.bfloat16, "W", 2)
    _need(y, torch.bfloat16, "y", 2)
    M, K = x.shape
    N = W.shape[0]
    if W.shape[1] != K:
        raise ValueError("W must be [N, K]")
    _shape(y, (M, N), "y")
    R = 0
    if A_cat is not None and A_cat.numel() > 0:
        _need(A_cat, torch.float32, "A_cat", 2)
        _need(B_cat, torch.float32, "B_cat", 2)
        R = A_cat.shape[0]
        if A_cat.shape[1] != K or tuple(B_cat.shape) != (N, R):
            raise ValueError("A_cat must be [R, K] and B_cat [N, R]")
    else:
        A_cat = B_cat = None
    _same_device(x, W, A_cat, B_cat, y)
    with torch.cuda.device(x.device):
        st = lib.lg_lora_linear_noalloc(_ptr(x), _ptr(W), _ptr(A_cat), _ptr(B_cat), _ptr(y), M, K, N, R,
                                        _stream(x.device))
    _check(st, "lg_lora_linear_noalloc")
    return y


def renoise(up, sigma, seed, offset=0, out=None):
    """x = (1 - sigma) up + sigma eps(seed, offset + i); FP32."""
    _need(up, torch.float32, "up")
    if out is None:
        out = torch.empty_like(up)
    _need(out, torch.float32, "out")
    if out.numel() != up.numel():
        raise ValueError("out must have as many elements as up")
    _same_device(up, out)
    with torch.cuda.device(up.device):
        st = lib.lg_renoise(_ptr(up), _ptr(out), up.numel(), float(sigma), int(seed), int(offset), _stream(up.device))
    _check(st, "lg_renoise")
    return out


def euler_step(x, v, sigma, sigma_next):
    """In place: x += (sigma_next - sigma) v; FP32."""
    _need(x, torch.float32, "x")
    _need(v, torch.float32, "v")
    if x.numel() != v.numel():
        raise ValueError("x and v must have the same number of elements")
    _same_device(x, v)
    with torch.cuda.device(x.device):
        st = lib.lg_euler_step(_ptr(x), _ptr(v), x.numel(), float(sigma), float(sigma_next), _stream(x.device))
    _check(st, "lg_euler_step")
    return x


# Routes of the IC sampler: printed start sigma on HyperFlow's eight-step,
# shift-12 table (page "Open-H3-Regenerate-2K-IC", section
# "三步接着放大的草稿画，八步从噪声重画").
IC_ROUTES = {"up3": 0.835, "up4": 0.923, "hf8": 1.0}


def shift_ladder(sigma0, n_steps=8, shift=12.0):
    """The FP32 sigmas a route visits: sigma0, then every point of the
    shift-`shift`, `n_steps`-step table below it (host computation)."""
    buf = (ctypes.c_float * (int(n_steps) + 2))()
    n = ctypes.c_int(0)
    st = lib.lg_shift_ladder(float(sigma0), int(n_steps), float(shift), buf, len(buf), ctypes.byref(n))
    _check(st, "lg_shift_ladder")
    return [float(buf[i]) for i in range(n.value)]


def philox_u32(n_blocks, seed, block_offset=0, out=None, device=None):
    """Raw Philox4x32-10 words, 4 per block, as an int32 tensor holding the uint32 bits."""
    if out is None:
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        out = torch.empty(4 * int(n_blocks), dtype=torch.int32, device=device)
    _need(out, torch.int32, "out")
    if out.numel() < 4 * n_blocks:
        raise ValueError("out too small")
    with torch.cuda.device(out.device):
        st = lib.lg_philox_u32(_ptr(out), int(n_blocks), int(seed), int(block_offset), _stream(out.device))
    _check(st, "lg_philox_u32")
    return out


def philox_normal(n, seed, offset=0, out=None, device=None):
    """eps[i] = element offset + i of the Box-Muller normal stream (FP32)."""
    if out is None:
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        out = torch.empty(int(n), dtype=torch.float32, device=device)
    _need(out, torch.float32, "out")
    if out.numel() < n:
        raise ValueError("out too small")
    with torch.cuda.device(out.device):
        st = lib.lg_philox_normal(_ptr(out), int(n), int(seed), int(offset), _stream(out.device))
    _check(st, "lg_philox_normal")
    return out
