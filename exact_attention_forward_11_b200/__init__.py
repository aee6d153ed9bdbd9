"""B200 (sm_100a) fused attention forward: Python binding of the C ABI.

The entry points below have the names and arguments of include/attn_b200.h and
only marshal arguments: every step of the computation runs in the CUDA kernels
of libattn_b200.so. There is no CPU fallback; if the library is missing the
calls raise. `forward`, `forward_from_host`, `quantize_fp8`, `forward_fp8`, `quantize_mxfp8`, `forward_mxfp8`,
`backward` and `w4a16_matmul` are torch conveniences
that allocate outputs with torch (PyTorch serves only for device memory and
streams) and call the same entry points.
"""
from __future__ import annotations

import ctypes
import math
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
RELEASE_LIB_PATH = os.path.join(_HERE, "libattn_b200.so")
# the debug build (device-side index checks, ATTN_ERR_BOUNDS): ATTN_B200_DEBUG=1
DEBUG_LIB_PATH = os.path.join(_HERE, "libattn_b200_debug.so")
LIB_PATH = DEBUG_LIB_PATH if os.environ.get("ATTN_B200_DEBUG", "0") not in ("", "0") else RELEASE_LIB_PATH

(ATTN_OK, ATTN_ERR_INVALID_ARG, ATTN_ERR_UNSUPPORTED, ATTN_ERR_MISALIGNED, ATTN_ERR_CUDA, ATTN_ERR_TIMEOUT,
 ATTN_ERR_BOUNDS) = range(7)
ATTN_BF16 = 0
TILE = 128

_lib = None

# (name, restype, argtypes) for every symbol the header declares
_P, _I, _F = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
SIGNATURES = {
    "attn_fwd": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _I, _P]),
    "attn_quantize_fp8": (_I, [_P, _P, _P, _P, _I, _I, _I, _I, _P]),
    "attn_fwd_fp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "attn_quantize_mxfp8": (_I, [_P, _P, _P, _I, _I, _I, _I, _P]),
    "attn_fwd_mxfp8": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "attn_get_device_status": (_I, [_P]),
    "attn_fwd_inject_timeout": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _I, ctypes.c_ulonglong, _P]),
    "attn_fwd_one_tile_inject_timeout": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _I, ctypes.c_ulonglong, _P]),
    "attn_bwd": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I, _I, _I, _I, _F, _I, _P]),
    "attn_bwd_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I, _I]),
    "attn_bwd_noalloc": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _P]),
    "w4a16_gemm": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _P]),
    "w4a16_gemm_splitk": (_I, [_P, _P, _P, _P, _P, _P, ctypes.c_size_t, _I, _I, _I, _P]),
    "w4a16_gemm_splitk_workspace_bytes": (ctypes.c_size_t, [_I, _I, _I]),
    "attn_fwd_mxfp8_inject_timeout": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, _I,
                                           ctypes.c_ulonglong, _P]),
    "attn_fwd_debug_row_limit": (_I, [_P, _P, _P, _P, _P, _I, _I, _I, _I, _F, _I, ctypes.c_longlong, _P]),
    "attn_debug_build": (_I, []),
    "attn_debug_last_failure": (_I, [ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_longlong), _P]),
    "attn_status_string": (ctypes.c_char_p, [_I]),
    "attn_abi_version": (_I, []),
}


class AttnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {attn_status_string(status)}")


def load():
    """Load the library at LIB_PATH: libattn_b200.so, or with ATTN_B200_DEBUG=1 its
    debug build libattn_b200_debug.so (both built by exact_attention_forward_11_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is not built: run `python -m exact_attention_forward_11_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


# ------------------------------------------------------------------ raw C ABI
def attn_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, dtype, stream):
    return load().attn_fwd(q, k, v, o, lse, B, H, N, d, scale, causal, dtype, stream)


def attn_quantize_fp8(x, rot, x8, scales, B, H, N, d, stream):
    return load().attn_quantize_fp8(x, rot, x8, scales, B, H, N, d, stream)


def attn_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, B, H, N, d, scale, causal, stream):
    return load().attn_fwd_fp8(q8, k8, v8, q_scale, k_scale, v_scale, o, lse, B, H, N, d, scale, causal, stream)


def attn_quantize_mxfp8(x, codes, sf, B, H, N, d, stream):
    return load().attn_quantize_mxfp8(x, codes, sf, B, H, N, d, stream)


def attn_fwd_mxfp8(q8, k8, v8, q_sf, k_sf, v_sf, o, lse, B, H, N, d, scale, causal, stream):
    return load().attn_fwd_mxfp8(q8, k8, v8, q_sf, k_sf, v_sf, o, lse, B, H, N, d, scale, causal, stream)


def attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, N, d, scale, causal, stream):
    return load().attn_bwd(q, k, v, o, lse, dout, dq, dk, dv, workspace, workspace_bytes, B, H, N, d, scale,
                           causal, stream)


def attn_bwd_workspace_bytes(B, H, N, d):
    return load().attn_bwd_workspace_bytes(B, H, N, d)


def w4a16_gemm(x, qweight, scales, zeros, y, M, N, K, stream):
    return load().w4a16_gemm(x, qweight, scales, zeros, y, M, N, K, stream)


def w4a16_gemm_splitk(x, qweight, scales, zeros, y, workspace, workspace_bytes, M, N, K, stream):
    return load().w4a16_gemm_splitk(x, qweight, scales, zeros, y, workspace, workspace_bytes, M, N, K, stream)


def w4a16_gemm_splitk_workspace_bytes(M, N, K):
    return load().w4a16_gemm_splitk_workspace_bytes(M, N, K)


def attn_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, stream):
    """attn_bwd with its scratch in a fixed array inside the library, for callers
    that cannot allocate device memory (include/attn_b200.h)."""
    return load().attn_bwd_noalloc(q, k, v, o, lse, dout, dq, dk, dv, B, H, N, d, scale, causal, stream)


ATTN_BWD_NOALLOC_MAX_ROWS = 1 << 21


def attn_fwd_inject_timeout(q, k, v, o, lse, B, H, N, d, scale, causal, fault_unit, wait_limit_cycles, stream):
    """Testing hook (include/attn_b200_testing.h): attn_fwd with one K tile withheld."""
    return load().attn_fwd_inject_timeout(q, k, v, o, lse, B, H, N, d, scale, causal, fault_unit,
                                          wait_limit_cycles, stream)


def attn_fwd_one_tile_inject_timeout(q, k, v, o, lse, B, H, N, d, scale, causal, fault_unit, wait_limit_cycles,
                                     stream):
    """Testing hook (include/attn_b200_testing.h): the one-Q-tile schedule with one K tile withheld."""
    return load().attn_fwd_one_tile_inject_timeout(q, k, v, o, lse, B, H, N, d, scale, causal, fault_unit,
                                                   wait_limit_cycles, stream)


def attn_fwd_mxfp8_inject_timeout(q8, k8, v8, q_sf, k_sf, v_sf, o, lse, B, H, N, d, scale, causal, fault_unit,
                                  wait_limit_cycles, stream):
    """Testing hook (include/attn_b200_testing.h): attn_fwd_mxfp8 with one K tile withheld."""
    return load().attn_fwd_mxfp8_inject_timeout(q8, k8, v8, q_sf, k_sf, v_sf, o, lse, B, H, N, d, scale, causal,
                                                fault_unit, wait_limit_cycles, stream)


def attn_fwd_debug_row_limit(q, k, v, o, lse, B, H, N, d, scale, causal, row_limit, stream):
    """Testing hook of the debug build (include/attn_b200_testing.h): attn_fwd told
    that O / LSE hold only `row_limit` rows."""
    return load().attn_fwd_debug_row_limit(q, k, v, o, lse, B, H, N, d, scale, causal, row_limit, stream)


def attn_debug_build():
    return load().attn_debug_build()


def attn_debug_last_failure(stream):
    """(site, index) of the first debug check that failed since the last call; site 0: none."""
    site, index = ctypes.c_int(0), ctypes.c_longlong(0)
    st = load().attn_debug_last_failure(ctypes.byref(site), ctypes.byref(index), stream)
    if st != ATTN_OK:
        raise AttnError(st, "attn_debug_last_failure")
    return site.value, index.value


def use_library(path):
    """Switch the binding to another build of the library (e.g. DEBUG_LIB_PATH);
    later calls go to it. Returns the previous path."""
    global _lib, LIB_PATH
    prev = LIB_PATH
    LIB_PATH = path
    _lib = None
    return prev


def attn_get_device_status(stream):
    st = load().attn_get_device_status(stream)
    if st != ATTN_OK and _W4_WORKSPACES:
        _reset_w4_workspaces()
    return st


def attn_status_string(status):
    return load().attn_status_string(int(status)).decode()


def attn_abi_version():
    return load().attn_abi_version()


# ------------------------------------------------------------------ torch helpers
def _stream_ptr(t, stream):
    import torch
    s = torch.cuda.current_stream(t.device) if stream is None else stream
    return s.cuda_stream


def _check(status, where):
    if status != ATTN_OK:
        raise AttnError(status, where)


def _ptr(t):
    return None if t is None else t.data_ptr()


def _shape4(q):
    if q.dim() != 4 or not q.is_contiguous() or not q.is_cuda:
        raise ValueError("expected a contiguous CUDA tensor [B, H, N, d]")
    return tuple(q.shape)


def _expect(t, name, shape, dtype, device):
    """Every tensor handed to the library must be a contiguous CUDA tensor of the
    exact shape and dtype, on the same device as the first input (the kernels
    read and write through raw device pointers)."""
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be a CUDA tensor on {device}")
    if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous {dtype} tensor of shape {tuple(shape)}")


def _check_device(check, stream_ptr, where):
    """With check=True, wait for the launch and read the library's device status
    word (one per device, shared by every stream and thread: a timeout of any
    earlier launch is reported here too)."""
    if check:
        _check(attn_get_device_status(stream_ptr), where + " (device status)")


def forward(q, k, v, causal=False, scale=None, out=None, lse=None, with_lse=True, stream=None, check=False):
    """O, LSE = attention(q, k, v) for bf16 CUDA tensors [B, H, N, d].

    The call is asynchronous. The outputs are valid once the launch has finished
    AND attn_get_device_status() reports ATTN_OK (a pipeline wait that timed out
    leaves them undefined); check=True does both before returning. `scale`
    None selects 1/sqrt(d); a negative scale raises AttnError."""
    import torch
    B, H, N, d = _shape4(q)
    for name, t in (("q", q), ("k", k), ("v", v)):
        _expect(t, name, (B, H, N, d), torch.bfloat16, q.device)
    if out is None:
        out = torch.empty_like(q)
    _expect(out, "out", (B, H, N, d), torch.bfloat16, q.device)
    if lse is None and with_lse:
        lse = torch.empty((B, H, N), device=q.device, dtype=torch.float32)
    if lse is not None:
        _expect(lse, "lse", (B, H, N), torch.float32, q.device)
    sc = 0.0 if scale is None else float(scale)
    sp = _stream_ptr(q, stream)
    _check(attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(), _ptr(lse), B, H, N, d, sc,
                    int(bool(causal)), ATTN_BF16, sp), "attn_fwd")
    _check_device(check, sp, "attn_fwd")
    return out, lse


_HOST_STREAMS = {}


def forward_from_host(q, k, v, causal=False, scale=None, out=None, lse=None, device=None, chunks=8):
    """O, LSE of attention for HOST tensors: bf16 [B, H, N, d] in (pinned) CPU
    memory in, O bf16 [B, H, N, d] and LSE fp32 [B, H, N] in (pinned) CPU memory
    out, for callers whose inputs arrive on the host.

    The B*H heads are cut into `chunks` contiguous groups (the heads are
    independent). Three streams overlap the copies with the kernels: group c+1
    is copied in while attn_fwd runs on group c (pointer offsets into the device
    buffers) and group c-1 is copied out, so the two PCIe directions and the GPU
    work at the same time. Returns once O and LSE are in host memory and the
    device status word reads ATTN_OK (raises AttnError otherwise). The results
    are the same bytes as forward() on the same inputs."""
    import torch

    from .sharded import head_range
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.is_cuda or t.dim() != 4 or not t.is_contiguous() or t.dtype != torch.bfloat16:
            raise ValueError(f"{name} must be a contiguous bf16 CPU tensor [B, H, N, d]")
    B, H, N, d = q.shape
    if k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v shapes differ")
    BH = B * H
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16).pin_memory()
    if lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32).pin_memory()
    if out.is_cuda or tuple(out.shape) != (B, H, N, d) or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 CPU tensor [B, H, N, d]")
    if lse.is_cuda or tuple(lse.shape) != (B, H, N) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 CPU tensor [B, H, N]")
    chunks = max(1, min(int(chunks), BH))
    key = dev.index
    if key not in _HOST_STREAMS:
        _HOST_STREAMS[key] = tuple(torch.cuda.Stream(dev) for _ in range(3))
    s_in, s_run, s_out = _HOST_STREAMS[key]
    flat = [t.view(BH, N, d) for t in (q, k, v)]
    o_flat, l_flat = out.view(BH, N, d), lse.view(BH, N)
    dq, dk, dv, do = (torch.empty((BH, N, d), dtype=torch.bfloat16, device=dev) for _ in range(4))
    # one LSE buffer per group: an offset of h0 * N floats into a shared one is
    # 16-byte aligned only when h0 * N is a multiple of 4
    dls = [torch.empty((head_range(BH, chunks, c)[1], N), dtype=torch.float32, device=dev) for c in range(chunks)]
    # the device buffers are allocated on the current stream; the three streams
    # start after it
    start = torch.cuda.Event()
    start.record(torch.cuda.current_stream(dev))
    for st in (s_in, s_run, s_out):
        st.wait_event(start)
    sc = 0.0 if scale is None else float(scale)
    elem = 2 * N * d
    for c in range(chunks):
        h0, cnt = head_range(BH, chunks, c)
        if cnt == 0:
            continue
        sl = slice(h0, h0 + cnt)
        with torch.cuda.stream(s_in):
            for dst, src in zip((dq, dk, dv), flat):
                dst[sl].copy_(src[sl], non_blocking=True)
            ready = torch.cuda.Event()
            ready.record(s_in)
        s_run.wait_event(ready)
        off = h0 * elem
        _check(attn_fwd(dq.data_ptr() + off, dk.data_ptr() + off, dv.data_ptr() + off, do.data_ptr() + off,
                        dls[c].data_ptr(), 1, cnt, N, d, sc, int(bool(causal)), ATTN_BF16,
                        s_run.cuda_stream), "attn_fwd")
        done = torch.cuda.Event()
        done.record(s_run)
        s_out.wait_event(done)
        with torch.cuda.stream(s_out):
            o_flat[sl].copy_(do[sl], non_blocking=True)
            l_flat[sl].copy_(dls[c], non_blocking=True)
    # every copy and launch above has finished once the copy-out stream has (it
    # waited on each group's kernel, which waited on that group's copies in), so
    # the device buffers can go back to the allocator when this returns
    s_out.synchronize()
    _check(attn_get_device_status(s_run.cuda_stream), "forward_from_host (device status)")
    return out, lse


def quantize_fp8(x, rot=None, stream=None):
    """(codes uint8 [B,H,N,d], scales fp32 [B,H,ceil(N/128)]) of a bf16 tensor."""
    import torch
    B, H, N, d = _shape4(x)
    _expect(x, "x", (B, H, N, d), torch.bfloat16, x.device)
    if rot is not None:
        _expect(rot, "rot", (d, d), torch.bfloat16, x.device)
    x8 = torch.empty((B, H, N, d), device=x.device, dtype=torch.uint8)
    scales = torch.empty((B, H, (N + TILE - 1) // TILE), device=x.device, dtype=torch.float32)
    _check(attn_quantize_fp8(x.data_ptr(), _ptr(rot), x8.data_ptr(), scales.data_ptr(), B, H, N, d,
                             _stream_ptr(x, stream)), "attn_quantize_fp8")
    return x8, scales


def forward_fp8(q8, k8, v8, q_scale, k_scale, v_scale, causal=False, scale=None, out=None, lse=None,
                with_lse=True, stream=None, check=False):
    """O (bf16), LSE from E4M3 codes and their per-tile scales (finite, >= 0).

    Asynchronous like forward(): the outputs are valid once the launch has
    finished and attn_get_device_status() reports ATTN_OK; check=True does both."""
    import torch
    B, H, N, d = _shape4(q8)
    T = (N + TILE - 1) // TILE
    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        _expect(t, name, (B, H, N, d), torch.uint8, q8.device)
    for name, t in (("q_scale", q_scale), ("k_scale", k_scale), ("v_scale", v_scale)):
        _expect(t, name, (B, H, T), torch.float32, q8.device)
    if out is None:
        out = torch.empty((B, H, N, d), device=q8.device, dtype=torch.bfloat16)
    _expect(out, "out", (B, H, N, d), torch.bfloat16, q8.device)
    if lse is None and with_lse:
        lse = torch.empty((B, H, N), device=q8.device, dtype=torch.float32)
    if lse is not None:
        _expect(lse, "lse", (B, H, N), torch.float32, q8.device)
    sc = 0.0 if scale is None else float(scale)
    sp = _stream_ptr(q8, stream)
    _check(attn_fwd_fp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), q_scale.data_ptr(), k_scale.data_ptr(),
                        v_scale.data_ptr(), out.data_ptr(), _ptr(lse), B, H, N, d, sc, int(bool(causal)), sp),
           "attn_fwd_fp8")
    _check_device(check, sp, "attn_fwd_fp8")
    return out, lse


def quantize_mxfp8(x, stream=None):
    """(codes uint8 [B,H,N,d], scale bytes uint8 [B,H,N,d/32]) of a bf16 tensor:
    MXFP8, one E8M0 scale per 32 consecutive values of a row."""
    import torch
    B, H, N, d = _shape4(x)
    _expect(x, "x", (B, H, N, d), torch.bfloat16, x.device)
    codes = torch.empty((B, H, N, d), device=x.device, dtype=torch.uint8)
    # the scale array is padded to 16 bytes so that its base stays 16-byte aligned
    nsf = B * H * N * (d // 32)
    sf = torch.empty(((nsf + 15) // 16) * 16, device=x.device, dtype=torch.uint8)[:nsf].view(B, H, N, d // 32)
    _check(attn_quantize_mxfp8(x.data_ptr(), codes.data_ptr(), sf.data_ptr(), B, H, N, d, _stream_ptr(x, stream)),
           "attn_quantize_mxfp8")
    return codes, sf


def forward_mxfp8(q8, k8, v8, q_sf, k_sf, v_sf, causal=False, scale=None, out=None, lse=None, with_lse=True,
                  stream=None, check=False):
    """O (bf16), LSE from MXFP8 codes [B,H,N,d] and their scale bytes [B,H,N,d/32].

    Asynchronous like forward(): the outputs are valid once the launch has
    finished and attn_get_device_status() reports ATTN_OK; check=True does both."""
    import torch
    B, H, N, d = _shape4(q8)
    for name, t in (("q8", q8), ("k8", k8), ("v8", v8)):
        _expect(t, name, (B, H, N, d), torch.uint8, q8.device)
    if d % 32:
        raise ValueError("d must be a multiple of 32")
    for name, t in (("q_sf", q_sf), ("k_sf", k_sf), ("v_sf", v_sf)):
        _expect(t, name, (B, H, N, d // 32), torch.uint8, q8.device)
    if out is None:
        out = torch.empty((B, H, N, d), device=q8.device, dtype=torch.bfloat16)
    _expect(out, "out", (B, H, N, d), torch.bfloat16, q8.device)
    if lse is None and with_lse:
        lse = torch.empty((B, H, N), device=q8.device, dtype=torch.float32)
    if lse is not None:
        _expect(lse, "lse", (B, H, N), torch.float32, q8.device)
    sc = 0.0 if scale is None else float(scale)
    sp = _stream_ptr(q8, stream)
    _check(attn_fwd_mxfp8(q8.data_ptr(), k8.data_ptr(), v8.data_ptr(), q_sf.data_ptr(), k_sf.data_ptr(),
                          v_sf.data_ptr(), out.data_ptr(), _ptr(lse), B, H, N, d, sc, int(bool(causal)), sp),
           "attn_fwd_mxfp8")
    _check_device(check, sp, "attn_fwd_mxfp8")
    return out, lse


def backward(q, k, v, o, lse, dout, causal=False, scale=None, dq=None, dk=None, dv=None, workspace=None,
             stream=None, check=False):
    """dQ, dK, dV of attention for bf16 CUDA tensors [B, H, N, d], given the
    forward's O and LSE and dout = dL/dO. The workspace (D_i per row) is
    allocated with torch unless given. Asynchronous like forward()."""
    import torch
    B, H, N, d = _shape4(q)
    for name, t in (("q", q), ("k", k), ("v", v), ("o", o), ("dout", dout)):
        _expect(t, name, (B, H, N, d), torch.bfloat16, q.device)
    _expect(lse, "lse", (B, H, N), torch.float32, q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(q) if dk is None else dk
    dv = torch.empty_like(q) if dv is None else dv
    for name, t in (("dq", dq), ("dk", dk), ("dv", dv)):
        _expect(t, name, (B, H, N, d), torch.bfloat16, q.device)
    need = attn_bwd_workspace_bytes(B, H, N, d)
    if need == 0:
        raise AttnError(ATTN_ERR_UNSUPPORTED, "attn_bwd_workspace_bytes")
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if not workspace.is_cuda or workspace.device != q.device or workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace must be a CUDA buffer of at least {need} bytes on {q.device}")
    sc = 0.0 if scale is None else float(scale)
    sp = _stream_ptr(q, stream)
    _check(attn_bwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dout.data_ptr(),
                    dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
                    workspace.numel() * workspace.element_size(), B, H, N, d, sc, int(bool(causal)), sp),
           "attn_bwd")
    _check_device(check, sp, "attn_bwd")
    return dq, dk, dv


# split-K workspaces of w4a16_matmul, one per (device, stream): zeroed when
# allocated; every call leaves the tickets zero again
_W4_WORKSPACES = {}


def _reset_w4_workspaces():
    """After a device status other than ATTN_OK a split-K call may have left
    tickets set: wait for the device and zero every cached workspace."""
    import torch
    torch.cuda.synchronize()
    for t in _W4_WORKSPACES.values():
        t.zero_()
    torch.cuda.synchronize()


def _w4_workspace(device, stream_ptr, nbytes):
    import torch
    key = (device.index, stream_ptr)
    ws = _W4_WORKSPACES.get(key)
    if ws is None or ws.numel() < nbytes:
        if ws is not None:
            torch.cuda.synchronize(device)        # the old one may still be read by a launch
        ws = torch.zeros(nbytes, dtype=torch.uint8, device=device)
        torch.cuda.current_stream(device).synchronize()   # zeroed before any stream uses it
        _W4_WORKSPACES[key] = ws
    return ws


def w4a16_matmul(x, qweight, scales, zeros, out=None, stream=None, check=False, split_k=True, workspace=None):
    """Y = X W for fp16 X [M, K] and W given as packed int4 (int32 [K/8, N]), fp16
    scales [K/128, N] and uint8 zero points [K/128, N] (include/w4a16_b200.h).

    split_k=True (default) runs w4a16_gemm_splitk, which balances the K slices over
    every SM; its workspace is `workspace` (a zeroed uint8 CUDA tensor of at least
    w4a16_gemm_splitk_workspace_bytes(M, N, K) bytes) or one cached per device and
    stream. split_k=False runs w4a16_gemm (one CTA per 128 output columns)."""
    import torch
    if x.dim() != 2:
        raise ValueError("x must be [M, K]")
    M, K = x.shape
    _expect(x, "x", (M, K), torch.float16, x.device)
    N = qweight.shape[1] if qweight.dim() == 2 else -1
    _expect(qweight, "qweight", (K // 8, N), torch.int32, x.device)
    _expect(scales, "scales", (K // 128, N), torch.float16, x.device)
    _expect(zeros, "zeros", (K // 128, N), torch.uint8, x.device)
    if out is None:
        out = torch.empty((M, N), dtype=torch.float16, device=x.device)
    _expect(out, "out", (M, N), torch.float16, x.device)
    sp = _stream_ptr(x, stream)
    if not split_k:
        _check(w4a16_gemm(x.data_ptr(), qweight.data_ptr(), scales.data_ptr(), zeros.data_ptr(), out.data_ptr(),
                          M, N, K, sp), "w4a16_gemm")
        _check_device(check, sp, "w4a16_gemm")
        return out
    need = w4a16_gemm_splitk_workspace_bytes(M, N, K)
    if need == 0:
        raise AttnError(ATTN_ERR_UNSUPPORTED, "w4a16_gemm_splitk_workspace_bytes")
    if workspace is None:
        workspace = _w4_workspace(x.device, sp, need)
    elif workspace.device != x.device or not workspace.is_contiguous() or \
            workspace.numel() * workspace.element_size() < need:
        raise ValueError(f"workspace must be a contiguous tensor of at least {need} bytes on {x.device}")
    _check(w4a16_gemm_splitk(x.data_ptr(), qweight.data_ptr(), scales.data_ptr(), zeros.data_ptr(),
                             out.data_ptr(), workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                             M, N, K, sp), "w4a16_gemm_splitk")
    _check_device(check, sp, "w4a16_gemm_splitk")
    return out


def flops(B, H, N, d, causal):
    """Algorithmic FLOPs of one forward: 4 B H N^2 d, halved for causal."""
    f = 4.0 * B * H * N * N * d
    return f / 2 if causal else f


def default_scale(d):
    return 1.0 / math.sqrt(d)
