"""Python binding of libfluxbin.so, the B200 LUT binary GEMV (C ABI in
include/fluxbin.h).

Argument marshalling only: every step of the computation runs in the CUDA
kernels of the library.  PyTorch supplies device memory and the current
stream.  If the compiled library is missing, importing the binding's
functions raises; there is no CPU fallback.

Names follow the C ABI: fb_pack, fb_pack_bits, fb_unpack, fb_vcm_gather,
fb_lut_build, fb_validate_weights, fb_gemv_workspace_bytes, fb_gemv,
fb_gemv_batched; ``Weights`` wraps one fb_weights struct and the tensors it
points to.
"""

from __future__ import annotations

import ctypes as C
import os
from typing import Optional, Tuple

import torch

__all__ = [
    "FbError", "Weights", "lib", "library_path", "FB_GEMV_PDL", "FB_GEMV_INDEPENDENT", "FB_GEMV_TEST_WAIT_TIMEOUT",
    "fb_packed_words", "fb_pack", "fb_pack_bits", "fb_unpack", "fb_vcm_gather",
    "fb_lut_build", "fb_validate_weights", "fb_gemv_workspace_bytes", "fb_gemv",
    "fb_gemv_batched", "fb_status_string", "fb_gemv_launch_plan", "fb_gemv_grouped", "fb_device_errors",
    "fb_fit_saliency", "fb_fit_base", "fit", "fb_gemv_group_scales",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_HERE, "libfluxbin.so")

FB_OK = 0
FB_GEMV_PDL = 1
FB_GEMV_INDEPENDENT = 2
FB_GEMV_TEST_WAIT_TIMEOUT = 0x80000000
_DTYPES = {torch.float32: 0, torch.float16: 1, torch.bfloat16: 2}
_STATUS = {0: "FB_OK", 1: "FB_ERR_INVALID_VALUE", 2: "FB_ERR_UNSUPPORTED", 3: "FB_ERR_MISALIGNED",
           4: "FB_ERR_WORKSPACE", 5: "FB_ERR_CUDA"}


class FbError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {_STATUS.get(status, status)}")


class FbWeightsStruct(C.Structure):
    _fields_ = [
        ("M", C.c_int), ("N", C.c_int), ("K", C.c_int), ("g", C.c_int),
        ("planes", C.c_void_p), ("alpha_r", C.c_void_p), ("alpha_c", C.c_void_p),
        ("nS", C.c_int), ("Ks", C.c_int),
        ("s_idx", C.c_void_p), ("s_planes", C.c_void_p),
        ("s_alpha_r", C.c_void_p), ("s_alpha_c", C.c_void_p),
    ]


_lib = None


def lib() -> C.CDLL:
    """The loaded C library, with argument types declared."""
    global _lib
    if _lib is None:
        if not os.path.exists(library_path):
            raise RuntimeError(
                f"{library_path} is missing: build it with `python -m lut_binary_gemv_b200.build` "
                "(nvcc, sm_100a). There is no CPU fallback.")
        L = C.CDLL(library_path)
        P, I, S = C.c_void_p, C.c_int, C.c_size_t
        W = C.POINTER(FbWeightsStruct)
        sig = {
            "fb_packed_words": (S, [I, I, I]),
            "fb_pack": (I, [P, I, I, I, P, P]),
            "fb_pack_bits": (I, [P, I, I, I, P, P]),
            "fb_unpack": (I, [P, I, I, I, P, P]),
            "fb_vcm_gather": (I, [P, I, I, I, I, P, I, I, P, I, P]),
            "fb_lut_build": (I, [P, I, P, I, I, I, P, P]),
            "fb_validate_weights": (I, [W]),
            "fb_gemv_workspace_bytes": (S, [W, I]),
            "fb_gemv": (I, [W, P, I, P, P, S, C.c_uint, P]),
            "fb_gemv_batched": (I, [W, P, I, I, I, P, I, P, S, C.c_uint, P]),
            "fb_gemv_launch_plan": (I, [W, I, C.c_uint, I, P]),
            "fb_gemv_grouped": (I, [P, I, P, I, P, C.c_uint, P]),
            "fb_gemv_group_scales": (I, [W, I, P, I, P, C.c_uint, P]),
            "fb_device_errors": (I, [P, I]),
            "fb_fit_saliency": (I, [P, I, I, I, P, I, I, I, P, P, P]),
            "fb_fit_base": (I, [P, I, I, I, I, P, I, P, P, P]),
            "fb_status_string": (C.c_char_p, [I]),
            "fb_abi_version": (I, []),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype, f.argtypes = res, args
        _lib = L
    return _lib


def _check(status: int, what: str):
    if status != FB_OK:
        raise FbError(status, what)


_raw_stream = getattr(torch._C, "_cuda_getCurrentRawStream", None)


def _stream(device: torch.device) -> int:
    """The current CUDA stream of `device` as a raw handle (the cheap
    accessor when torch has it: eager calls are bound by host time)."""
    if _raw_stream is not None:
        return _raw_stream(device.index if device.index is not None else torch.cuda.current_device())
    return torch.cuda.current_stream(device).cuda_stream


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def fb_status_string(status: int) -> str:
    return lib().fb_status_string(status).decode()


def fb_packed_words(K: int, M: int, N: int) -> int:
    return lib().fb_packed_words(K, M, N)


def _new_planes(K, M, N, device):
    n = fb_packed_words(K, M, N)
    if n == 0:
        raise FbError(1, "fb_packed_words")
    return torch.empty(n, dtype=torch.int32, device=device)


def fb_pack(signs: torch.Tensor, planes: Optional[torch.Tensor] = None) -> torch.Tensor:
    """signs: int8 [K, M, N] (+1/-1) on the GPU -> packed planes (int32 words)."""
    K, M, N = signs.shape
    signs = signs.contiguous()
    planes = _new_planes(K, M, N, signs.device) if planes is None else planes
    _check(lib().fb_pack(signs.data_ptr(), K, M, N, planes.data_ptr(), _stream(signs.device)), "fb_pack")
    return planes


def fb_pack_bits(bits: torch.Tensor, N: int, planes: Optional[torch.Tensor] = None) -> torch.Tensor:
    """bits: uint8 [K, M, N/8] canonical bit planes on the GPU -> packed planes."""
    K, M, nb = bits.shape
    if nb * 8 != N:
        raise ValueError("bits must have N/8 bytes per row")
    bits = bits.contiguous()
    planes = _new_planes(K, M, N, bits.device) if planes is None else planes
    _check(lib().fb_pack_bits(bits.data_ptr(), K, M, N, planes.data_ptr(), _stream(bits.device)),
           "fb_pack_bits")
    return planes


def fb_unpack(planes: torch.Tensor, K: int, M: int, N: int) -> torch.Tensor:
    signs = torch.empty((K, M, N), dtype=torch.int8, device=planes.device)
    _check(lib().fb_unpack(planes.data_ptr(), K, M, N, signs.data_ptr(), _stream(planes.device)), "fb_unpack")
    return signs


def fb_vcm_gather(src: torch.Tensor, s_idx: torch.Tensor, nS_pad: int) -> torch.Tensor:
    """src: [nvec, n_src] (f32/f16/bf16); s_idx: int32 [nS] -> [nvec, nS_pad]."""
    src2 = src.reshape(-1, src.shape[-1]) if src.dim() != 1 else src.reshape(1, -1)
    nvec, n_src = src2.shape
    if src2.stride(-1) != 1:
        src2 = src2.contiguous()
    nS = s_idx.numel()
    dst = torch.empty((nvec, nS_pad), dtype=src.dtype, device=src.device)
    _check(lib().fb_vcm_gather(src2.data_ptr(), _DTYPES[src.dtype], nvec, n_src, src2.stride(0),
                               _ptr(s_idx) if nS else None, nS, nS_pad, dst.data_ptr(), nS_pad,
                               _stream(src.device)), "fb_vcm_gather")
    return dst if src.dim() != 1 else dst.reshape(-1)


def fb_lut_build(x: torch.Tensor, alpha_c: Optional[torch.Tensor], K: int, g: int) -> torch.Tensor:
    """LUT-BSF tables [K, N/g, 2^g] fp32 for one activation vector x [N]."""
    x = x.contiguous()
    N = x.numel()
    lut = torch.empty((K, N // g, 1 << g), dtype=torch.float32, device=x.device)
    ac = None if alpha_c is None else alpha_c.contiguous()
    _check(lib().fb_lut_build(x.data_ptr(), _DTYPES[x.dtype], _ptr(ac), K, N, g, lut.data_ptr(),
                              _stream(x.device)), "fb_lut_build")
    return lut


class Weights:
    """One fb_weights struct plus the device tensors it points to."""

    def __init__(self, M: int, N: int, K: int, g: int, planes: torch.Tensor, alpha_r: torch.Tensor,
                 alpha_c: Optional[torch.Tensor] = None, nS: int = 0, Ks: int = 0,
                 s_idx: Optional[torch.Tensor] = None, s_planes: Optional[torch.Tensor] = None,
                 s_alpha_r: Optional[torch.Tensor] = None, s_alpha_c: Optional[torch.Tensor] = None):
        self.M, self.N, self.K, self.g, self.nS, self.Ks = M, N, K, g, nS, Ks if nS else 0
        self.planes, self.alpha_r, self.alpha_c = planes, alpha_r, alpha_c
        self.s_idx, self.s_planes, self.s_alpha_r, self.s_alpha_c = s_idx, s_planes, s_alpha_r, s_alpha_c
        self.device = planes.device
        self.struct = FbWeightsStruct(
            M=M, N=N, K=K, g=g, planes=_ptr(planes), alpha_r=_ptr(alpha_r), alpha_c=_ptr(alpha_c),
            nS=nS, Ks=self.Ks, s_idx=_ptr(s_idx) if nS else None, s_planes=_ptr(s_planes) if nS else None,
            s_alpha_r=_ptr(s_alpha_r) if nS else None, s_alpha_c=_ptr(s_alpha_c) if nS else None)

    @property
    def ref(self):
        ref = self.__dict__.get("_ref")
        if ref is None:
            ref = self._ref = C.byref(self.struct)
        return ref

    def with_g(self, g: int) -> "Weights":
        """The same tensors with another LUT group width (the packed layout
        does not depend on g)."""
        return Weights(self.M, self.N, self.K, g, self.planes, self.alpha_r, self.alpha_c, self.nS,
                       self.Ks, self.s_idx, self.s_planes, self.s_alpha_r, self.s_alpha_c)

    @classmethod
    def from_arrays(cls, M, N, K, g, sign_bits, alpha_r, alpha_c=None, s_idx=None, s_sign_bits=None,
                    s_alpha_r=None, s_alpha_c=None, device="cuda") -> "Weights":
        """Upload canonical bit planes and scales (numpy or torch) and pack them on the GPU."""
        dev = torch.device(device)

        def up(a, dtype=None):
            if a is None:
                return None
            t = torch.as_tensor(a)
            if dtype is not None:
                t = t.to(dtype)
            return t.to(dev).contiguous()

        planes = fb_pack_bits(up(sign_bits, torch.uint8), N)
        nS = 0 if s_idx is None else len(s_idx)
        kw = {}
        if nS:
            nS_pad = (nS + 31) // 32 * 32
            kw = dict(nS=nS, Ks=int(s_alpha_r.shape[0]),
                      s_idx=up(torch.as_tensor(s_idx).to(torch.int64).to(torch.int32)),
                      s_planes=fb_pack_bits(up(s_sign_bits, torch.uint8), nS_pad),
                      s_alpha_r=up(s_alpha_r, torch.float32), s_alpha_c=up(s_alpha_c, torch.float32))
        return cls(M, N, K, g, planes, up(alpha_r, torch.float32), up(alpha_c, torch.float32), **kw)

    @classmethod
    def from_problem(cls, p, device="cuda", g: Optional[int] = None) -> "Weights":
        """From a workloads.Problem (its canonical arrays)."""
        return cls.from_arrays(p.M, p.N, p.K, p.g if g is None else g, p.sign_bits, p.alpha_r, p.alpha_c,
                               p.s_idx if p.nS else None, p.s_sign_bits, p.s_alpha_r, p.s_alpha_c,
                               device=device)


def fb_validate_weights(W: Weights) -> int:
    return lib().fb_validate_weights(W.ref)


def fb_gemv_workspace_bytes(W: Weights, batch: int = 1) -> int:
    return lib().fb_gemv_workspace_bytes(W.ref, batch)


def fb_gemv(W: Weights, x: torch.Tensor, y: Optional[torch.Tensor] = None,
            ws: Optional[torch.Tensor] = None, flags: int = 0) -> torch.Tensor:
    """y = W_hat x for one activation vector x [N] (f32/f16/bf16) -> fp32 [M]."""
    if x.stride(-1) != 1:
        x = x.contiguous()
    y = torch.empty(W.M, dtype=torch.float32, device=x.device) if y is None else y
    # the kernels need no workspace (fb_gemv_workspace_bytes is 0): NULL, 0 unless one is given
    wp, wn = (None, 0) if ws is None else (ws.data_ptr(), ws.numel() * ws.element_size())
    _check(lib().fb_gemv(W.ref, x.data_ptr(), _DTYPES[x.dtype], y.data_ptr(), wp, wn, flags,
                         _stream(x.device)), "fb_gemv")
    return y


def fb_gemv_batched(W: Weights, X: torch.Tensor, Y: Optional[torch.Tensor] = None,
                    ws: Optional[torch.Tensor] = None, flags: int = 0) -> torch.Tensor:
    """Y[b] = W_hat X[b] for X [B, N] -> fp32 [B, M]."""
    B = X.shape[0]
    if X.stride(-1) != 1:
        X = X.contiguous()
    Y = torch.empty((B, W.M), dtype=torch.float32, device=X.device) if Y is None else Y
    wp, wn = (None, 0) if ws is None else (ws.data_ptr(), ws.numel() * ws.element_size())
    _check(lib().fb_gemv_batched(W.ref, X.data_ptr(), _DTYPES[X.dtype], B, X.stride(0), Y.data_ptr(),
                                 Y.stride(0), wp, wn, flags, _stream(X.device)), "fb_gemv_batched")
    return Y


def fb_gemv_launch_plan(W, batch: int = 1, flags: int = 0, sms: int = 148) -> dict:
    """The launch shape fb_gemv would use for W (a Weights or an
    FbWeightsStruct: only its sizes and pointer alignment are read, so no GPU
    is needed)."""
    out = (C.c_int * 6)()
    ref = W.ref if isinstance(W, Weights) else C.byref(W)
    _check(lib().fb_gemv_launch_plan(ref, batch, flags, sms, C.cast(out, C.c_void_p)), "fb_gemv_launch_plan")
    return dict(zip(("C", "cpb", "RB", "warps", "smem", "V"), list(out)))


def fb_device_errors(clear: bool = True) -> int:
    """Error bits raised by GEMV kernels since the last clear (synchronises the device)."""
    flags = C.c_uint(0)
    _check(lib().fb_device_errors(C.cast(C.byref(flags), C.c_void_p), int(clear)), "fb_device_errors")
    return flags.value


def fb_gemv_grouped(Ws, x: torch.Tensor, ys=None, flags: int = 0):
    """One launch for up to 4 matrices of one format that read the same x
    (q/k/v, gate/up): returns [y_m] with y_m = W_hat_m x."""
    n = len(Ws)
    if ys is None:
        ys = [torch.empty(W.M, dtype=torch.float32, device=x.device) for W in Ws]
    wp = (C.POINTER(FbWeightsStruct) * n)(*[C.pointer(W.struct) for W in Ws])
    yp = (C.c_void_p * n)(*[y.data_ptr() for y in ys])
    _check(lib().fb_gemv_grouped(C.cast(wp, C.c_void_p), n, x.data_ptr(), _DTYPES[x.dtype],
                                 C.cast(yp, C.c_void_p), flags, _stream(x.device)), "fb_gemv_grouped")
    return ys


def fb_gemv_group_scales(W: Weights, G: int, x: torch.Tensor, alpha_r_groups: torch.Tensor,
                         y: Optional[torch.Tensor] = None, flags: int = 0) -> torch.Tensor:
    """y = W_hat x with one row scale per group of G input columns:
    alpha_r_groups fp32 [K, N/G, M] (replacing W.alpha_r); W's other tensors
    as for fb_gemv."""
    if x.stride(-1) != 1:
        x = x.contiguous()
    if G <= 0 or W.N % G:
        raise ValueError("G must be a positive divisor of N")
    if (alpha_r_groups.dtype != torch.float32 or not alpha_r_groups.is_contiguous()
            or alpha_r_groups.numel() != W.K * (W.N // G) * W.M):
        raise ValueError("alpha_r_groups: contiguous float32 [K, N/G, M]")
    y = torch.empty(W.M, dtype=torch.float32, device=x.device) if y is None else y
    st = FbWeightsStruct.from_buffer_copy(W.struct)
    st.alpha_r = alpha_r_groups.data_ptr()
    _check(lib().fb_gemv_group_scales(C.byref(st), G, x.data_ptr(), _DTYPES[x.dtype], y.data_ptr(), flags,
                                      _stream(x.device)), "fb_gemv_group_scales")
    return y


def _f32_rows(t: torch.Tensor, what: str) -> torch.Tensor:
    if t.dim() != 2 or t.dtype != torch.float32 or t.stride(1) != 1:
        raise ValueError(f"{what}: a float32 matrix with unit column stride")
    return t


def fb_fit_saliency(W: torch.Tensor, X: torch.Tensor, nS: int) -> Tuple[torch.Tensor, torch.Tensor]:
    """Column scores (diagonal-Hessian proxy) and the nS salient columns.
    W [M, N], X [T, N] fp32 on the GPU -> (score fp32 [N], s_idx int32 [nS],
    ascending)."""
    W, X = _f32_rows(W, "W"), _f32_rows(X, "X")
    M, N = W.shape
    T = X.shape[0]
    if X.shape[1] != N:
        raise ValueError("X must have W's columns")
    score = torch.empty(N, dtype=torch.float32, device=W.device)
    s_idx = torch.empty(max(nS, 0), dtype=torch.int32, device=W.device)
    _check(lib().fb_fit_saliency(W.data_ptr(), M, N, W.stride(0), X.data_ptr(), T, X.stride(0), nS,
                                 score.data_ptr(), s_idx.data_ptr() if nS > 0 else None, _stream(W.device)),
           "fb_fit_saliency")
    return score, s_idx


def fb_fit_base(R: torch.Tensor, sweeps: int, signs: Optional[torch.Tensor] = None,
                alpha_r: Optional[torch.Tensor] = None,
                alpha_c: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """One greedy base on the residual R [M, N] fp32 (updated in place) ->
    (signs int8 [M, N], alpha_r fp32 [M], alpha_c fp32 [N]), written into the
    given outputs when passed (signs: unit column stride; scales contiguous)."""
    R = _f32_rows(R, "R")
    M, N = R.shape
    signs = torch.empty((M, N), dtype=torch.int8, device=R.device) if signs is None else signs
    ar = torch.empty(M, dtype=torch.float32, device=R.device) if alpha_r is None else alpha_r
    ac = torch.empty(N, dtype=torch.float32, device=R.device) if alpha_c is None else alpha_c
    if (signs.shape != (M, N) or signs.dtype != torch.int8 or signs.stride(1) != 1 or ar.shape != (M,)
            or ac.shape != (N,) or not ar.is_contiguous() or not ac.is_contiguous()):
        raise ValueError("fb_fit_base: output shapes")
    _check(lib().fb_fit_base(R.data_ptr(), M, N, R.stride(0), sweeps, signs.data_ptr(), signs.stride(0),
                             ar.data_ptr(), ac.data_ptr(), _stream(R.device)), "fb_fit_base")
    return signs, ar, ac


def fit(W: torch.Tensor, X: torch.Tensor, K: int, Ks: int, nS: int, sweeps: int) -> dict:
    """The whole fit on the GPU: K global bases on R = W, then the salient
    set and Ks bases on the residual's salient columns (gathered by
    fb_vcm_gather, padded to a multiple of 32 with zero columns).  Returns
    signs [K, M, N], alpha_r [K, M], alpha_c [K, N], score [N], s_idx [nS],
    s_signs [Ks, M, nS], s_alpha_r [Ks, M], s_alpha_c [Ks, nS], residual
    [M, N] (after the global bases) and s_residual [M, nS] (after the salient
    ones)."""
    W = _f32_rows(W, "W")
    M, N = W.shape
    dev = W.device
    score, s_idx = fb_fit_saliency(W, X, nS)
    R = W.clone()
    signs = torch.empty((K, M, N), dtype=torch.int8, device=dev)
    ar = torch.empty((K, M), dtype=torch.float32, device=dev)
    ac = torch.empty((K, N), dtype=torch.float32, device=dev)
    for k in range(K):
        fb_fit_base(R, sweeps, signs[k], ar[k], ac[k])
    nS_pad = (nS + 31) // 32 * 32
    # the salient bases run over the padded gather (zero columns past nS);
    # the views below drop the padding
    s_signs = torch.empty((Ks, M, nS_pad), dtype=torch.int8, device=dev)
    s_ar = torch.empty((Ks, M), dtype=torch.float32, device=dev)
    s_ac = torch.empty((Ks, nS_pad), dtype=torch.float32, device=dev)
    RS = None
    if nS > 0 and Ks > 0:
        RS = fb_vcm_gather(R, s_idx, nS_pad)
        for k in range(Ks):
            fb_fit_base(RS, sweeps, s_signs[k], s_ar[k], s_ac[k])
    return {"signs": signs, "alpha_r": ar, "alpha_c": ac, "score": score, "s_idx": s_idx,
            "s_signs": s_signs[:, :, :nS], "s_alpha_r": s_ar, "s_alpha_c": s_ac[:, :nS], "residual": R,
            "s_residual": None if RS is None else RS[:, :nS]}
