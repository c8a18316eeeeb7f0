"""Python binding of the B200 FP8 block-scaled NT GEMM library (libdg.so).

Argument marshalling only: every function here forwards torch tensors' device
pointers, their sizes and the current CUDA stream to the C ABI of
``include/dg.h`` with the same name.  All arithmetic runs in the sm_100a kernels
of ``libdg.so``; there is no fallback.  If the library is missing the first call
raises ``RuntimeError`` (build it with ``__graft_entry__.build()`` or
``python -m moe_grouped_gemm_weight_b200.build``).

Layouts (see include/dg.h):
  A   uint8 / float8_e4m3fn [M, K]          (masked: [G, M_max, K])
  sa  float32, transposed: sa[kb*sa_stride + m] (masked: per group blocks)
  B   uint8 / float8_e4m3fn [N, K] or [G, N, K]
  sb  float32 [ceil(N/128), K/128] or [G, ceil(N/128), K/128]
  D   bfloat16 [M, N]                        (masked: [G, M_max, N])
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libdg.so")

DG_OK, DG_ERR_INVALID_ARG, DG_ERR_UNSUPPORTED, DG_ERR_MISALIGNED, DG_ERR_CUDA = range(5)
DG_DEVERR_TIMEOUT, DG_DEVERR_BAD_M_INDEX, DG_DEVERR_BAD_MASKED_M, DG_DEVERR_NOT_POW2 = 1, 2, 4, 8
DG_DEVERR_BAD_K_OFFSET = 16

_lock = threading.Lock()
_lib = None


class DGError(RuntimeError):
    def __init__(self, func: str, status: int, message: str):
        super().__init__(f"{func}: {message} (status {status})")
        self.status = status


class Plan(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in
                ("block_m", "block_n", "stages", "m_blocks", "n_blocks", "tiles", "grid", "smem_bytes",
                 "swap_ab", "split_k", "tail_split")]

    def as_dict(self) -> dict:
        return {n: getattr(self, n) for n, _ in self._fields_}


def lib() -> ctypes.CDLL:
    """The loaded libdg.so (raises RuntimeError if it has not been built)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"CUDA library {LIB_PATH} is missing: run __graft_entry__.build() first")
            L = ctypes.CDLL(LIB_PATH)
            P, I = ctypes.c_void_p, ctypes.c_int
            L.dg_fp8_gemm_nt.restype = I
            L.dg_fp8_gemm_nt.argtypes = [P, P, P, I, P, P, I, I, I, P]
            for nm in ("dg_fp8_gemm_nn", "dg_fp8_gemm_tn", "dg_fp8_gemm_tt"):
                getattr(L, nm).restype = I
                getattr(L, nm).argtypes = [P, P, P, I, P, P, I, I, I, P]
            L.dg_k_grouped_fp8_gemm_tn.restype = I
            L.dg_k_grouped_fp8_gemm_tn.argtypes = [P, P, P, I, P, P, P, I, I, I, I, P]
            L.dg_fp8_gemm_nt_ue8m0.restype = I
            L.dg_fp8_gemm_nt_ue8m0.argtypes = [P, P, P, I, P, P, I, I, I, P]
            L.dg_fp8_gemm_nt_noalloc.restype = I
            L.dg_fp8_gemm_nt_noalloc.argtypes = [P, P, P, I, P, P, I, I, I, P]
            L.dg_to_fp8_1x128.restype = I
            L.dg_to_fp8_1x128.argtypes = [P, P, I, P, I, I, P]
            L.dg_to_fp8_128x128.restype = I
            L.dg_to_fp8_128x128.argtypes = [P, P, P, I, I, P]
            L.dg_grouped_contiguous_nt.restype = I
            L.dg_grouped_contiguous_nt.argtypes = [P, P, P, I, P, P, P, I, I, I, I, P]
            L.dg_grouped_masked_nt.restype = I
            L.dg_grouped_masked_nt.argtypes = [P, P, P, I, P, P, P, I, I, I, I, I, P]
            L.dg_set_pdl.restype = None
            L.dg_set_pdl.argtypes = [I]
            L.dg_get_pdl.restype = I
            L.dg_get_pdl.argtypes = []
            L.dg_set_num_sms.restype = None
            L.dg_set_num_sms.argtypes = [I]
            L.dg_get_num_sms.restype = I
            L.dg_get_num_sms.argtypes = []
            L.dg_get_m_alignment_for_contiguous_layout.restype = I
            L.dg_get_m_alignment_for_contiguous_layout.argtypes = []
            L.dg_get_tma_aligned_size.restype = I
            L.dg_get_tma_aligned_size.argtypes = [I, I]
            L.dg_get_device_error.restype = I
            L.dg_get_device_error.argtypes = [ctypes.POINTER(I)]
            L.dg_get_workspace_count.restype = I
            L.dg_get_workspace_count.argtypes = []
            L.dg_status_string.restype = ctypes.c_char_p
            L.dg_status_string.argtypes = [I]
            L.dg_last_error_message.restype = ctypes.c_char_p
            L.dg_last_error_message.argtypes = []
            L.dg_selftest_bounded_wait.restype = I
            L.dg_selftest_bounded_wait.argtypes = [P]
            L.dg_make_plan.restype = I
            L.dg_make_plan.argtypes = [I, I, I, I, I, I, ctypes.POINTER(Plan)]
            L.dg_make_plan_ue8m0.restype = I
            L.dg_make_plan_ue8m0.argtypes = [I, I, I, I, ctypes.POINTER(Plan)]
            _lib = L
    return _lib


def _check(func: str, status: int) -> None:
    if status != DG_OK:
        L = lib()
        msg = L.dg_last_error_message().decode() or L.dg_status_string(status).decode()
        raise DGError(func, status, msg)


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _cdiv(a: int, b: int) -> int:
    return -(-a // b)


def _sa_need(kblocks: int, sa_stride: int, rows: int) -> int:
    """Elements of a transposed scale array sa[kb*sa_stride + m] that the
    library touches for kb < kblocks, m < rows."""
    return 0 if kblocks <= 0 or rows <= 0 else (kblocks - 1) * int(sa_stride) + rows


def _check_dim(func: str, what: str, got: int, want: int) -> None:
    if got != want:
        raise DGError(func, DG_ERR_INVALID_ARG, f"{what} is {got}, expected {want}")


def _check_args(func: str, *specs) -> None:
    """Check the tensor arguments before their pointers cross the C boundary.

    Each spec is (name, tensor, element bytes, elements the call touches).  The
    C ABI takes plain device pointers and cannot see extents, so a tensor that
    is too short, strided, of another element type, or not on the current CUDA
    device would be read or written outside its memory by the kernels.  Such a
    call raises DGError (DG_ERR_INVALID_ARG) here and launches nothing.  None
    passes through: the library itself reports a null pointer."""
    given = [sp for sp in specs if sp[1] is not None]
    for name, t, esize, need in given:
        if t.element_size() != esize:
            raise DGError(func, DG_ERR_INVALID_ARG,
                          f"{name} has {t.element_size()}-byte elements, the call takes {esize}-byte ones")
        if not t.is_contiguous():
            raise DGError(func, DG_ERR_INVALID_ARG, f"{name} is not contiguous")
        if t.numel() < need:
            raise DGError(func, DG_ERR_INVALID_ARG, f"{name} holds {t.numel()} elements, the call touches {need}")
    for name, t, _, _ in given:
        if t.device.type != "cuda":
            raise DGError(func, DG_ERR_INVALID_ARG, f"{name} is not on a CUDA device ({t.device})")
    if given:
        import torch
        cur = torch.cuda.current_device()
        for name, t, _, _ in given:
            if t.device.index != cur:
                raise DGError(func, DG_ERR_INVALID_ARG, f"{name} is on {t.device}, the current device is cuda:{cur}")


def _check_dense(func: str, D, A, sa, sa_stride, B, sb, M: int, N: int, K: int, b_k: int) -> None:
    """Arguments of a dense call: D [M][N] bf16, A with M*K codes, sa
    transposed per 1x128, B with N*K codes (its K extent b_k), sb
    [ceil(N/128)][K/128]."""
    _check_dim(func, "K of B", b_k, K)
    nkb = _cdiv(K, 128)
    _check_args(func, ("D", D, 2, M * N), ("A", A, 1, M * K), ("sa", sa, 4, _sa_need(nkb, sa_stride, M)),
                ("B", B, 1, N * K), ("sb", sb, 4, _cdiv(N, 128) * nkb))


def _stream(stream) -> int:
    if stream is None:
        import torch
        return int(torch.cuda.current_stream().cuda_stream)
    return int(stream if isinstance(stream, int) else stream.cuda_stream)


def dg_fp8_gemm_nt(D, A, sa, sa_stride: int, B, sb, stream=None) -> None:
    """Dense D[M,N] = scaled A[M,K] . B[N,K]^T (sizes taken from A and B)."""
    M, K = A.shape[-2], A.shape[-1]
    N = B.shape[-2]
    _check_dense("dg_fp8_gemm_nt", D, A, sa, sa_stride, B, sb, M, N, K, B.shape[-1])
    _check("dg_fp8_gemm_nt", lib().dg_fp8_gemm_nt(_ptr(D), _ptr(A), _ptr(sa), int(sa_stride), _ptr(B), _ptr(sb),
                                                  M, N, K, _stream(stream)))


def dg_fp8_gemm_nn(D, A, sa, sa_stride: int, B, sb, stream=None) -> None:
    """D[M,N] = scaled A . B^T with A [M,K] and B stored [K,N]."""
    M, K = A.shape[-2], A.shape[-1]
    N = B.shape[-1]
    _check_dense("dg_fp8_gemm_nn", D, A, sa, sa_stride, B, sb, M, N, K, B.shape[-2])
    _check("dg_fp8_gemm_nn", lib().dg_fp8_gemm_nn(_ptr(D), _ptr(A), _ptr(sa), int(sa_stride), _ptr(B), _ptr(sb),
                                                  M, N, K, _stream(stream)))


def dg_fp8_gemm_tn(D, A, sa, sa_stride: int, B, sb, stream=None) -> None:
    """D[M,N] = scaled A . B^T with A stored [K,M] and B stored [K,N]."""
    K, M = A.shape[-2], A.shape[-1]
    N = B.shape[-1]
    _check_dense("dg_fp8_gemm_tn", D, A, sa, sa_stride, B, sb, M, N, K, B.shape[-2])
    _check("dg_fp8_gemm_tn", lib().dg_fp8_gemm_tn(_ptr(D), _ptr(A), _ptr(sa), int(sa_stride), _ptr(B), _ptr(sb),
                                                  M, N, K, _stream(stream)))


def dg_fp8_gemm_tt(D, A, sa, sa_stride: int, B, sb, stream=None) -> None:
    """D[M,N] = scaled A . B^T with A stored [K,M] and B [N,K]."""
    K, M = A.shape[-2], A.shape[-1]
    N = B.shape[-2]
    _check_dense("dg_fp8_gemm_tt", D, A, sa, sa_stride, B, sb, M, N, K, B.shape[-1])
    _check("dg_fp8_gemm_tt", lib().dg_fp8_gemm_tt(_ptr(D), _ptr(A), _ptr(sa), int(sa_stride), _ptr(B), _ptr(sb),
                                                  M, N, K, _stream(stream)))


def dg_k_grouped_fp8_gemm_tn(D, A, sa, sa_stride: int, B, sb, k_offsets, stream=None) -> None:
    """K-grouped GEMM: A stored [K,M], B stored [K,N], k_offsets int32 [G+1] on the
    device, D [G,M,N]."""
    K, M = A.shape[-2], A.shape[-1]
    N = B.shape[-1]
    G = k_offsets.numel() - 1
    func = "dg_k_grouped_fp8_gemm_tn"
    _check_dim(func, "K of B", B.shape[-2], K)
    nkb = _cdiv(K, 128)
    _check_args(func, ("D", D, 2, max(G, 0) * M * N), ("A", A, 1, M * K), ("sa", sa, 4, _sa_need(nkb, sa_stride, M)),
                ("B", B, 1, N * K), ("sb", sb, 4, _cdiv(N, 128) * nkb), ("k_offsets", k_offsets, 4, G + 1))
    _check("dg_k_grouped_fp8_gemm_tn",
           lib().dg_k_grouped_fp8_gemm_tn(_ptr(D), _ptr(A), _ptr(sa), int(sa_stride), _ptr(B), _ptr(sb),
                                          _ptr(k_offsets), G, M, N, K, _stream(stream)))


def dg_fp8_gemm_nt_ue8m0(D, A, sa, sa_stride: int, B, sb, stream=None) -> None:
    """dg_fp8_gemm_nt for power-of-two sa / sb, scaled inside the tensor core."""
    M, K = A.shape[-2], A.shape[-1]
    N = B.shape[-2]
    _check_dense("dg_fp8_gemm_nt_ue8m0", D, A, sa, sa_stride, B, sb, M, N, K, B.shape[-1])
    _check("dg_fp8_gemm_nt_ue8m0", lib().dg_fp8_gemm_nt_ue8m0(_ptr(D), _ptr(A), _ptr(sa), int(sa_stride), _ptr(B),
                                                            _ptr(sb), M, N, K, _stream(stream)))


def dg_fp8_gemm_nt_noalloc(D, A, sa, sa_stride: int, B, sb, stream=None) -> None:
    """dg_fp8_gemm_nt without device allocation: the K-split scratch is a static
    16 MiB array shared by every call on the device, so calls that overlap on
    the GPU race.  Make the first call on each device before any stream capture."""
    M, K = A.shape[-2], A.shape[-1]
    N = B.shape[-2]
    _check_dense("dg_fp8_gemm_nt_noalloc", D, A, sa, sa_stride, B, sb, M, N, K, B.shape[-1])
    _check("dg_fp8_gemm_nt_noalloc",
           lib().dg_fp8_gemm_nt_noalloc(_ptr(D), _ptr(A), _ptr(sa), int(sa_stride), _ptr(B), _ptr(sb),
                                        M, N, K, _stream(stream)))


def dg_to_fp8_1x128(Q, sa, sa_stride: int, X, stream=None) -> None:
    """Activation cast: bf16 X [M,K] -> e4m3 Q [M,K] (uint8) and sa[kb*sa_stride + m]."""
    M, K = X.shape[-2], X.shape[-1]
    _check_args("dg_to_fp8_1x128", ("Q", Q, 1, M * K), ("sa", sa, 4, _sa_need(_cdiv(K, 128), sa_stride, M)),
                ("X", X, 2, M * K))
    _check("dg_to_fp8_1x128", lib().dg_to_fp8_1x128(_ptr(Q), _ptr(sa), int(sa_stride), _ptr(X), M, K,
                                                    _stream(stream)))


def dg_to_fp8_128x128(Q, sb, W, stream=None) -> None:
    """Weight cast: bf16 W [N,K] -> e4m3 Q [N,K] (uint8) and sb [ceil(N/128), K/128]."""
    N, K = W.shape[-2], W.shape[-1]
    _check_args("dg_to_fp8_128x128", ("Q", Q, 1, N * K), ("sb", sb, 4, _cdiv(N, 128) * _cdiv(K, 128)),
                ("W", W, 2, N * K))
    _check("dg_to_fp8_128x128", lib().dg_to_fp8_128x128(_ptr(Q), _ptr(sb), _ptr(W), N, K, _stream(stream)))


def dg_grouped_contiguous_nt(D, A, sa, sa_stride: int, B, sb, m_indices, stream=None) -> None:
    """Contiguous-layout grouped GEMM; B is [G,N,K], m_indices int32 [M_total]."""
    M, K = A.shape[-2], A.shape[-1]
    func = "dg_grouped_contiguous_nt"
    _check_dim(func, "rank of B", B.dim(), 3)
    G, N = B.shape[0], B.shape[1]
    _check_dim(func, "K of B", B.shape[2], K)
    nkb = _cdiv(K, 128)
    _check_args(func, ("D", D, 2, M * N), ("A", A, 1, M * K), ("sa", sa, 4, _sa_need(nkb, sa_stride, M)),
                ("B", B, 1, G * N * K), ("sb", sb, 4, G * _cdiv(N, 128) * nkb), ("m_indices", m_indices, 4, M))
    _check("dg_grouped_contiguous_nt",
           lib().dg_grouped_contiguous_nt(_ptr(D), _ptr(A), _ptr(sa), int(sa_stride), _ptr(B), _ptr(sb),
                                          _ptr(m_indices), M, N, K, G, _stream(stream)))


def dg_grouped_masked_nt(D, A, sa, sa_stride: int, B, sb, masked_m, expected_m: int = 0, stream=None) -> None:
    """Masked-layout grouped GEMM; A is [G,M_max,K], masked_m int32 [G] on the device."""
    func = "dg_grouped_masked_nt"
    _check_dim(func, "rank of A", A.dim(), 3)
    _check_dim(func, "rank of B", B.dim(), 3)
    G, Mmax, K = A.shape
    N = B.shape[1]
    _check_dim(func, "group count of B", B.shape[0], G)
    _check_dim(func, "K of B", B.shape[2], K)
    nkb = _cdiv(K, 128)
    _check_args(func, ("D", D, 2, G * Mmax * N), ("A", A, 1, G * Mmax * K),
                ("sa", sa, 4, _sa_need(G * nkb, sa_stride, Mmax)), ("B", B, 1, G * N * K),
                ("sb", sb, 4, G * _cdiv(N, 128) * nkb), ("masked_m", masked_m, 4, G))
    _check("dg_grouped_masked_nt",
           lib().dg_grouped_masked_nt(_ptr(D), _ptr(A), _ptr(sa), int(sa_stride), _ptr(B), _ptr(sb),
                                      _ptr(masked_m), G, Mmax, N, K, int(expected_m), _stream(stream)))


def dg_set_pdl(enable) -> None:
    """Programmatic dependent launch on (True), off (False) or default (None: DG_PDL=1)."""
    lib().dg_set_pdl(-1 if enable is None else int(bool(enable)))


def dg_get_pdl() -> bool:
    return bool(lib().dg_get_pdl())


def dg_set_num_sms(n: int) -> None:
    lib().dg_set_num_sms(int(n))


def dg_get_num_sms() -> int:
    return int(lib().dg_get_num_sms())


def dg_get_m_alignment_for_contiguous_layout() -> int:
    return int(lib().dg_get_m_alignment_for_contiguous_layout())


def dg_get_tma_aligned_size(x: int, elem_bytes: int) -> int:
    return int(lib().dg_get_tma_aligned_size(int(x), int(elem_bytes)))


def dg_get_device_error() -> int:
    code = ctypes.c_int(0)
    _check("dg_get_device_error", lib().dg_get_device_error(ctypes.byref(code)))
    return int(code.value)


def dg_get_workspace_count() -> int:
    return int(lib().dg_get_workspace_count())


def dg_make_plan(mode: int, rows: int, N: int, K: int, G: int, num_sms: int) -> dict:
    pl = Plan()
    _check("dg_make_plan", lib().dg_make_plan(int(mode), int(rows), int(N), int(K), int(G), int(num_sms),
                                              ctypes.byref(pl)))
    return pl.as_dict()


def dg_make_plan_ue8m0(M: int, N: int, K: int, num_sms: int) -> dict:
    pl = Plan()
    _check("dg_make_plan_ue8m0", lib().dg_make_plan_ue8m0(int(M), int(N), int(K), int(num_sms), ctypes.byref(pl)))
    return pl.as_dict()


def dg_selftest_bounded_wait(stream=None) -> None:
    """Enqueue the bounded-wait self-test kernel (sets DG_DEVERR_TIMEOUT after ~1 s)."""
    _check("dg_selftest_bounded_wait", lib().dg_selftest_bounded_wait(_stream(stream)))


def dg_status_string(status: int) -> str:
    return lib().dg_status_string(int(status)).decode()


def dg_get_col_major_tma_aligned_tensor(s):
    """[M, nkb] (or [G, M, nkb]) float32 scales -> (flat transposed TMA-aligned tensor, sa_stride).

    Layout helper for callers (the pages' get_col_major_tma_aligned_tensor);
    runs as torch tensor ops outside the timed path."""
    import torch
    grouped = s.dim() == 3
    s3 = s if grouped else s.unsqueeze(0)
    G, M, nkb = s3.shape
    stride = dg_get_tma_aligned_size(M, 4)
    out = torch.zeros(G, nkb, stride, dtype=torch.float32, device=s.device)
    out[:, :, :M] = s3.transpose(1, 2)
    return out.reshape(-1).contiguous(), stride
