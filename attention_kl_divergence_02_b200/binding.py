"""ctypes binding of libstreamkl (include/streamkl.h).

Argument marshalling only: torch tensors are turned into device pointers and the CUDA
stream handle, and every step of the computation runs in the library's kernels.  The
library is loaded on first use; if it is missing or fails to load this raises, there is
no other implementation to fall back to.

Low-level functions carry the C names and arguments (pointers may be ints or tensors).
``fwd``/``bwd`` are conveniences that allocate outputs with torch (device memory is
torch's job; the library allocates nothing).
"""
import ctypes
import math
import os

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libstreamkl.so")

OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED = 2
ERR_CUDA = 3
ERR_TIMEOUT = 4

EXPORTS = (
    "streamkl_fwd",
    "streamkl_fwd_sym",
    "streamkl_fwd_splitk",
    "streamkl_fwd_splits",
    "streamkl_fwd_splitk_workspace_bytes",
    "streamkl_bwd",
    "streamkl_bwd_workspace_bytes",
    "streamkl_bwd_noalloc",
    "streamkl_status_string",
    "streamkl_device_status",
    "streamkl_selftest_watchdog",
    "streamkl_last_cuda_error",
    "streamkl_version",
    "streamkl_probe_exp2",
    "streamkl_num_sms",
    "streamkl_probe_clock",
    "streamkl_eval_exp2",
)

_lib = None


class StreamKLError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        msg = "%s: %s" % (where, status_string(status))
        if status == ERR_CUDA:
            msg += " (%s)" % last_cuda_error()
        super().__init__(msg)


def load(path=None):
    """Load the shared library (once) and declare the C signatures."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise ImportError("libstreamkl.so not built at %s (run python -m "
                          "attention_kl_divergence_02_b200.build)" % p)
    lib = ctypes.CDLL(p)
    vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    lib.streamkl_fwd.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, vp, vp, vp]
    lib.streamkl_fwd.restype = i
    lib.streamkl_fwd_sym.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, vp, vp, vp, vp]
    lib.streamkl_fwd_sym.restype = i
    lib.streamkl_fwd_splitk.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, vp, vp, vp, vp, sz, vp]
    lib.streamkl_fwd_splitk.restype = i
    lib.streamkl_fwd_splits.argtypes = [i, i, i, i]
    lib.streamkl_fwd_splits.restype = i
    lib.streamkl_fwd_splitk_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.streamkl_fwd_splitk_workspace_bytes.restype = sz
    lib.streamkl_bwd.argtypes = ([i, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i,
                                  vp, vp, vp, sz, vp])
    lib.streamkl_bwd.restype = i
    lib.streamkl_bwd_noalloc.argtypes = ([i, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i,
                                          vp, vp, vp])
    lib.streamkl_bwd_noalloc.restype = i
    lib.streamkl_bwd_workspace_bytes.argtypes = [i, i, i, i, i, i]
    lib.streamkl_bwd_workspace_bytes.restype = sz
    lib.streamkl_status_string.argtypes = [i]
    lib.streamkl_status_string.restype = ctypes.c_char_p
    lib.streamkl_device_status.argtypes = [vp]
    lib.streamkl_device_status.restype = i
    lib.streamkl_selftest_watchdog.argtypes = [i, ctypes.POINTER(ctypes.c_longlong), vp]
    lib.streamkl_selftest_watchdog.restype = i
    lib.streamkl_last_cuda_error.argtypes = []
    lib.streamkl_last_cuda_error.restype = ctypes.c_char_p
    lib.streamkl_version.argtypes = []
    lib.streamkl_version.restype = i
    lib.streamkl_probe_exp2.argtypes = [i, i, ctypes.POINTER(ctypes.c_longlong), vp]
    lib.streamkl_probe_exp2.restype = i
    lib.streamkl_num_sms.argtypes = []
    lib.streamkl_num_sms.restype = i
    lib.streamkl_probe_clock.argtypes = [ctypes.c_longlong, ctypes.c_longlong, vp, i, vp]
    lib.streamkl_probe_clock.restype = i
    lib.streamkl_eval_exp2.argtypes = [i, vp, vp, ctypes.c_longlong, vp]
    lib.streamkl_eval_exp2.restype = i
    if path is None:
        _lib = lib
    return lib


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


# ------------------------------------------------------------------ C-named calls
def streamkl_fwd(q1, k1, q2, k2, B, Hq, Hkv, NQ, NK, d, scale, causal, kl, lse1, lse2, stream=None):
    return load().streamkl_fwd(_ptr(q1), _ptr(k1), _ptr(q2), _ptr(k2), B, Hq, Hkv, NQ, NK, d,
                               float(scale), int(bool(causal)), _ptr(kl), _ptr(lse1), _ptr(lse2),
                               _stream(stream))


def streamkl_fwd_sym(q1, k1, q2, k2, B, Hq, Hkv, NQ, NK, d, scale, causal, kl12, kl21, lse1, lse2,
                     stream=None):
    return load().streamkl_fwd_sym(_ptr(q1), _ptr(k1), _ptr(q2), _ptr(k2), B, Hq, Hkv, NQ, NK, d,
                                   float(scale), int(bool(causal)), _ptr(kl12), _ptr(kl21), _ptr(lse1),
                                   _ptr(lse2), _stream(stream))


def streamkl_fwd_splitk(q1, k1, q2, k2, B, Hq, Hkv, NQ, NK, d, scale, causal, splits, kl, lse1, lse2,
                        workspace, workspace_bytes, stream=None):
    return load().streamkl_fwd_splitk(_ptr(q1), _ptr(k1), _ptr(q2), _ptr(k2), B, Hq, Hkv, NQ, NK, d,
                                      float(scale), int(bool(causal)), int(splits), _ptr(kl),
                                      _ptr(lse1), _ptr(lse2), _ptr(workspace), int(workspace_bytes),
                                      _stream(stream))


def streamkl_fwd_splits(B, Hq, NQ, NK):
    return load().streamkl_fwd_splits(B, Hq, NQ, NK)


def streamkl_fwd_splitk_workspace_bytes(B, Hq, NQ, NK, splits):
    return load().streamkl_fwd_splitk_workspace_bytes(B, Hq, NQ, NK, splits)


def streamkl_bwd(mode, q1, k1, q2, k2, kl, lse1, lse2, dkl, B, Hq, Hkv, NQ, NK, d, scale, causal,
                 dq, dk, workspace, workspace_bytes, stream=None):
    return load().streamkl_bwd(int(mode), _ptr(q1), _ptr(k1), _ptr(q2), _ptr(k2), _ptr(kl),
                               _ptr(lse1), _ptr(lse2), _ptr(dkl), B, Hq, Hkv, NQ, NK, d,
                               float(scale), int(bool(causal)), _ptr(dq), _ptr(dk),
                               _ptr(workspace), int(workspace_bytes), _stream(stream))


# Built-in scratch of streamkl_bwd_noalloc (STREAMKL_NOALLOC_SCRATCH_BYTES in the header).
NOALLOC_SCRATCH_BYTES = 32 << 20


def streamkl_bwd_noalloc(mode, q1, k1, q2, k2, kl, lse1, lse2, dkl, B, Hq, Hkv, NQ, NK, d, scale,
                         causal, dq, dk, stream=None):
    """Backward without a workspace argument, for callers that may not allocate device
    memory: the library's fixed 32 MiB built-in buffer holds what streamkl_bwd keeps in its
    workspace (the dK accumulator, plus the dQ partial sums when keys are split into ranges),
    so sizes with streamkl_bwd_workspace_bytes(...) > 32 MiB return ERR_UNSUPPORTED.  Calls
    that can overlap on the GPU share that buffer and race."""
    return load().streamkl_bwd_noalloc(int(mode), _ptr(q1), _ptr(k1), _ptr(q2), _ptr(k2), _ptr(kl),
                                       _ptr(lse1), _ptr(lse2), _ptr(dkl), B, Hq, Hkv, NQ, NK, d,
                                       float(scale), int(bool(causal)), _ptr(dq), _ptr(dk),
                                       _stream(stream))


def streamkl_bwd_workspace_bytes(B, Hq, Hkv, NQ, NK, d):
    return load().streamkl_bwd_workspace_bytes(B, Hq, Hkv, NQ, NK, d)


def streamkl_device_status(stream=None):
    return load().streamkl_device_status(_stream(stream))


def streamkl_selftest_watchdog(starve, stream=None):
    """Runs the bounded-wait self-test; returns (status, [ns of wait 0, ns of wait 1])."""
    ns = (ctypes.c_longlong * 2)()
    rc = load().streamkl_selftest_watchdog(int(starve), ns, _stream(stream))
    return rc, [ns[0], ns[1]]


def streamkl_probe_exp2(kind, iters, stream=None):
    """Launches the exponential-throughput probe; returns (status, exponentials evaluated)."""
    n = ctypes.c_longlong(0)
    rc = load().streamkl_probe_exp2(int(kind), int(iters), ctypes.byref(n), _stream(stream))
    return rc, n.value


def streamkl_num_sms():
    return load().streamkl_num_sms()


def streamkl_probe_clock(duration_ns, interval_ns, samples, stream=None):
    """Launches the clock probe into `samples` (int64 device tensor of 2 + 2 * max_pairs
    elements); returns the status."""
    import torch
    if samples.dtype != torch.int64 or not samples.is_cuda or not samples.is_contiguous() \
            or samples.numel() < 6:
        raise ValueError("samples must be a contiguous int64 CUDA tensor of at least 6 elements")
    n = samples.numel()
    return load().streamkl_probe_clock(int(duration_ns), int(interval_ns), _ptr(samples),
                                       int((n - 2) // 2), _stream(stream))


def streamkl_eval_exp2(kind, x, stream=None):
    """2^x by the kernels' exponential path `kind` (0: exponential unit, 1: FMA-pipe
    polynomial) for a contiguous fp32 CUDA tensor; returns (status, y)."""
    import torch
    if x.dtype != torch.float32 or not x.is_cuda or not x.is_contiguous():
        raise ValueError("x must be a contiguous fp32 CUDA tensor")
    y = torch.empty_like(x)
    rc = load().streamkl_eval_exp2(int(kind), _ptr(x), _ptr(y), x.numel(), _stream(stream))
    return rc, y


def status_string(status):
    return load().streamkl_status_string(int(status)).decode()


def last_cuda_error():
    return load().streamkl_last_cuda_error().decode()


def version():
    return load().streamkl_version()


# ------------------------------------------------------------------ conveniences
def _dims(q1, k1):
    B, Hq, NQ, d = q1.shape
    _, Hkv, NK, _ = k1.shape
    return B, Hq, Hkv, NQ, NK, d


def _check_inputs(q1, k1, q2, k2):
    """Refuses inputs whose shapes or devices disagree: the library sizes every tensor map
    from q1's batch and head dimension and k1's key count, so a mismatch would make a kernel
    read past an allocation."""
    import torch
    for t in (q1, k1, q2, k2):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError("inputs must be contiguous bf16 CUDA tensors")
    if q1.dim() != 4 or k1.dim() != 4 or q1.shape != q2.shape or k1.shape != k2.shape:
        raise ValueError("q1/q2 must be [B,Hq,NQ,d], k1/k2 [B,Hkv,NK,d]")
    if q1.shape[0] != k1.shape[0] or q1.shape[3] != k1.shape[3]:
        raise ValueError("q and k must share batch size and head dim (q %s, k %s)"
                         % (tuple(q1.shape), tuple(k1.shape)))
    if k1.shape[1] < 1 or q1.shape[1] % k1.shape[1] != 0:
        raise ValueError("query heads (%d) must be a multiple of KV heads (%d)"
                         % (q1.shape[1], k1.shape[1]))
    if len({t.device for t in (q1, k1, q2, k2)}) != 1:
        raise ValueError("q1, k1, q2, k2 must be on one device")


def _check_tensor(name, t, shape, dtype, device):
    """Refuses a tensor the kernels would read or write out of bounds or misinterpret."""
    if t is None:
        raise ValueError("%s is required" % name)
    if t.dtype != dtype or t.device != device or not t.is_contiguous() or tuple(t.shape) != tuple(shape):
        raise ValueError("%s must be a contiguous %s tensor of shape %s on %s (got %s %s on %s)"
                         % (name, dtype, tuple(shape), device, t.dtype, tuple(t.shape), t.device))


def _check_workspace(workspace, nbytes, device):
    if workspace.device != device or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous tensor on %s" % device)
    have = workspace.numel() * workspace.element_size()
    if have < nbytes:
        raise ValueError("workspace holds %d bytes, %d needed" % (have, nbytes))


def fwd(q1, k1, q2, k2, scale=None, causal=False, out=None, stream=None):
    """Returns (kl, lse1, lse2), fp32 [B,Hq,NQ].  Pass k2 = k1 (same tensor) for shared keys."""
    import torch
    _check_inputs(q1, k1, q2, k2)
    B, Hq, Hkv, NQ, NK, d = _dims(q1, k1)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is None:
        out = tuple(torch.empty((B, Hq, NQ), dtype=torch.float32, device=q1.device) for _ in range(3))
    for name, o in zip(("kl", "lse1", "lse2"), out):
        _check_tensor(name, o, (B, Hq, NQ), torch.float32, q1.device)
    rc = streamkl_fwd(q1, k1, q2, k2, B, Hq, Hkv, NQ, NK, d, scale, causal, *out, stream=stream)
    if rc != OK:
        raise StreamKLError(rc, "streamkl_fwd")
    return out


def fwd_sym(q1, k1, q2, k2, scale=None, causal=False, out=None, stream=None):
    """Returns (kl12, kl21, lse1, lse2), fp32 [B,Hq,NQ]: KL(P1||P2), KL(P2||P1) and both LSEs in
    one pass over the keys; kl12 + kl21 is the symmetric divergence."""
    import torch
    _check_inputs(q1, k1, q2, k2)
    B, Hq, Hkv, NQ, NK, d = _dims(q1, k1)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is None:
        out = tuple(torch.empty((B, Hq, NQ), dtype=torch.float32, device=q1.device) for _ in range(4))
    for name, o in zip(("kl12", "kl21", "lse1", "lse2"), out):
        _check_tensor(name, o, (B, Hq, NQ), torch.float32, q1.device)
    rc = streamkl_fwd_sym(q1, k1, q2, k2, B, Hq, Hkv, NQ, NK, d, scale, causal, *out, stream=stream)
    if rc != OK:
        raise StreamKLError(rc, "streamkl_fwd_sym")
    return out


def fwd_splitk(q1, k1, q2, k2, scale=None, causal=False, splits=0, out=None, workspace=None,
               stream=None):
    """Split-K forward (key ranges merged exactly); same outputs as fwd.  splits = 0 lets
    the library choose; `workspace` (fp32 tensor) is allocated here when not given."""
    import torch
    _check_inputs(q1, k1, q2, k2)
    B, Hq, Hkv, NQ, NK, d = _dims(q1, k1)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    if out is None:
        out = tuple(torch.empty((B, Hq, NQ), dtype=torch.float32, device=q1.device) for _ in range(3))
    for name, o in zip(("kl", "lse1", "lse2"), out):
        _check_tensor(name, o, (B, Hq, NQ), torch.float32, q1.device)
    need = streamkl_fwd_splitk_workspace_bytes(B, Hq, NQ, NK, splits)
    if workspace is None and need > 0:
        workspace = torch.empty((need + 3) // 4, dtype=torch.float32, device=q1.device)
    if workspace is not None:
        _check_workspace(workspace, need, q1.device)
    wbytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    rc = streamkl_fwd_splitk(q1, k1, q2, k2, B, Hq, Hkv, NQ, NK, d, scale, causal, splits, *out,
                             workspace, wbytes, stream=stream)
    if rc != OK:
        raise StreamKLError(rc, "streamkl_fwd_splitk")
    return out


def bwd(mode, q1, k1, q2, k2, kl, lse1, lse2, dkl, scale=None, causal=False, out=None,
        workspace=None, stream=None):
    """Returns (dq, dk) of the free distribution: mode 1 -> (dQ2, dK2), mode 2 -> (dQ1, dK1)."""
    import torch
    _check_inputs(q1, k1, q2, k2)
    B, Hq, Hkv, NQ, NK, d = _dims(q1, k1)
    scale = 1.0 / math.sqrt(d) if scale is None else scale
    for name, v in zip(("kl", "lse1", "lse2", "dkl"), (kl, lse1, lse2, dkl)):
        _check_tensor(name, v, (B, Hq, NQ), torch.float32, q1.device)
    if out is None:
        out = (torch.empty_like(q1), torch.empty_like(k1))
    _check_tensor("dq", out[0], q1.shape, torch.bfloat16, q1.device)
    _check_tensor("dk", out[1], k1.shape, torch.bfloat16, q1.device)
    nbytes = streamkl_bwd_workspace_bytes(B, Hq, Hkv, NQ, NK, d)
    if workspace is None:
        workspace = torch.empty(max(nbytes, 16) // 4, dtype=torch.float32, device=q1.device)
    _check_workspace(workspace, nbytes, q1.device)
    rc = streamkl_bwd(mode, q1, k1, q2, k2, kl, lse1, lse2, dkl, B, Hq, Hkv, NQ, NK, d, scale,
                      causal, out[0], out[1], workspace, workspace.numel() * workspace.element_size(),
                      stream=stream)
    if rc != OK:
        raise StreamKLError(rc, "streamkl_bwd")
    return out
