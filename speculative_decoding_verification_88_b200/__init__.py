"""speculative_decoding_verification_88_b200 -- verify-and-accept for
speculative decoding on B200 (sm_100a).

A thin ctypes binding over ``libspecverify.so`` (C ABI in
``include/spec_verify.h``).  PyTorch is used only for device memory and
streams: every step of the verify path runs in the library's CUDA kernels.
There is no CPU fallback; calls raise if the library or a CUDA device is
missing.

    import speculative_decoding_verification_88_b200 as sv
    r = sv.stochastic(target, draft, draft_tokens, temperature=0.7, seed=1)
    r["accepted_len"], r["out_tokens"]
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

from .build import LIB_PATH

SV_F32, SV_BF16 = 0, 1
SV_FLAG_INVALID_TOKEN, SV_FLAG_RESIDUAL_FALLBACK, SV_FLAG_TIMEOUT = 1, 2, 4
SV_FLAG_INVALID_ROW, SV_FLAG_CAPACITY, SV_FLAG_INVALID_TREE = 8, 16, 32
SV_FLAG_BOUNDS = 64  # raised by the bounds-checked build only

# Entry points declared in include/spec_verify.h.
EXPORTS = (
    "spec_verify_workspace_size", "spec_verify_status_string", "spec_verify_workspace_init",
    "spec_verify_read_device_status", "spec_verify_stochastic", "spec_verify_greedy",
    "spec_verify_multi_candidate", "spec_verify_multi_candidate_rows", "spec_verify_commit",
    "spec_verify_tree_workspace_size", "spec_verify_tree_greedy", "spec_verify_threshold",
    "spec_verify_philox4x32_10", "spec_verify_greedy_noalloc",
    "spec_verify_greedy_noalloc_read_device_status",
    "spec_verify_tree_stochastic_workspace_size", "spec_verify_tree_stochastic",
    "spec_verify_kernel_launches",
)

_lib = None
_lock = threading.Lock()


class SpecVerifyError(RuntimeError):
    pass


def library_path() -> str:
    return LIB_PATH


def load_library(path: str | None = None):
    """Load libspecverify.so (raises if it has not been built).  `path` loads
    another build of the same library (the bounds-checked one) and returns it
    without making it the default."""
    global _lib
    with _lock:
        if path is None and _lib is not None:
            return _lib
        target = path or LIB_PATH
        if not os.path.exists(target):
            raise SpecVerifyError(
                f"{target} is missing: build it with "
                "`python -m speculative_decoding_verification_88_b200.build`")
        lib = ctypes.CDLL(target)
        P, I, I64, U32, U64, SZ, F = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                                      ctypes.c_uint32, ctypes.c_uint64, ctypes.c_size_t,
                                      ctypes.c_float)
        lib.spec_verify_workspace_size.argtypes = [I, I, I, I]
        lib.spec_verify_workspace_size.restype = SZ
        lib.spec_verify_status_string.argtypes = [I]
        lib.spec_verify_status_string.restype = ctypes.c_char_p
        lib.spec_verify_workspace_init.argtypes = [P, SZ, P]
        lib.spec_verify_workspace_init.restype = I
        lib.spec_verify_read_device_status.argtypes = [P, ctypes.POINTER(U32), I, P]
        lib.spec_verify_read_device_status.restype = I
        lib.spec_verify_stochastic.argtypes = [
            P, I, I64, I64, P, I, I64, I64, P, I, I, I, F, U64, U32, P, P, P, P, SZ, P]
        lib.spec_verify_stochastic.restype = I
        lib.spec_verify_greedy.argtypes = [P, I, I64, I64, P, I, I, I, P, P, P, SZ, P]
        lib.spec_verify_greedy.restype = I
        lib.spec_verify_multi_candidate.argtypes = [
            P, I, I64, I64, I64, P, I, I, I, I, P, P, P, P, SZ, P]
        lib.spec_verify_multi_candidate.restype = I
        lib.spec_verify_multi_candidate_rows.argtypes = [
            P, I, I64, I64, P, P, I, I, I, I, I, P, P, P, P, SZ, P]
        lib.spec_verify_multi_candidate_rows.restype = I
        lib.spec_verify_commit.argtypes = [P, P, I, I, P, P, I64, I, P, P, P]
        lib.spec_verify_commit.restype = I
        lib.spec_verify_tree_workspace_size.argtypes = [I, I, I]
        lib.spec_verify_tree_workspace_size.restype = SZ
        lib.spec_verify_tree_greedy.argtypes = [P, I, I64, I64, P, P, I, I, I, P, P, P, P, SZ, P]
        lib.spec_verify_tree_greedy.restype = I
        lib.spec_verify_threshold.argtypes = [P, I, I64, I64, P, I, I, I, F, F, P, P, P, SZ, P]
        lib.spec_verify_threshold.restype = I
        lib.spec_verify_tree_stochastic_workspace_size.argtypes = [I, I, I]
        lib.spec_verify_tree_stochastic_workspace_size.restype = SZ
        lib.spec_verify_tree_stochastic.argtypes = [
            P, I, I64, I64, P, P, I, I, I, F, U64, U32, P, P, P, P, SZ, P]
        lib.spec_verify_tree_stochastic.restype = I
        lib.spec_verify_philox4x32_10.argtypes = [P, I64, U64, P, P]
        lib.spec_verify_philox4x32_10.restype = I
        lib.spec_verify_greedy_noalloc.argtypes = [P, I, I64, I64, P, I, I, I, P, P, P]
        lib.spec_verify_greedy_noalloc.restype = I
        lib.spec_verify_greedy_noalloc_read_device_status.argtypes = [ctypes.POINTER(U32), I, P]
        lib.spec_verify_greedy_noalloc_read_device_status.restype = I
        lib.spec_verify_kernel_launches.argtypes = []
        lib.spec_verify_kernel_launches.restype = U64
        if path is None:
            _lib = lib
        return lib


def status_string(code: int) -> str:
    return load_library().spec_verify_status_string(int(code)).decode()


def _check(code: int, what: str):
    if code != 0:
        raise SpecVerifyError(f"{what}: {status_string(code)}")


def launch_count() -> int:
    """Kernels the library has launched in this process so far (its own
    count; a launch captured into a CUDA graph counts once, at capture)."""
    return int(load_library().spec_verify_kernel_launches())


def workspace_size(B: int, G: int, k: int, V: int) -> int:
    return int(load_library().spec_verify_workspace_size(B, G, k, V))


class Workspace:
    """A zero-initialised device workspace, grown on demand (one per stream)."""

    def __init__(self, device=None, nbytes: int = 0):
        self.device = torch.device(device if device is not None else "cuda")
        self.buf = None
        self.ensure(nbytes)

    @property
    def nbytes(self) -> int:
        return 0 if self.buf is None else self.buf.numel()

    def ensure(self, nbytes: int, stream=None):
        if nbytes <= self.nbytes:
            return self
        self.buf = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=self.device)
        _check(load_library().spec_verify_workspace_init(
            self.buf.data_ptr(), self.buf.numel(), _stream_ptr(stream, self.device)),
            "spec_verify_workspace_init")
        return self

    def reset(self, stream=None):
        if self.buf is not None:
            _check(load_library().spec_verify_workspace_init(
                self.buf.data_ptr(), self.buf.numel(), _stream_ptr(stream, self.device)),
                "spec_verify_workspace_init")

    def device_status(self, clear: bool = True, stream=None) -> int:
        """Sticky SV_FLAG_* bits of the device (synchronises the stream)."""
        v = ctypes.c_uint32(0)
        _check(load_library().spec_verify_read_device_status(
            self.buf.data_ptr(), ctypes.byref(v), int(clear), _stream_ptr(stream, self.device)),
            "spec_verify_read_device_status")
        return int(v.value)


_default_ws: dict = {}


def default_workspace(device) -> Workspace:
    key = (torch.device(device), torch.cuda.current_stream(device).cuda_stream)
    ws = _default_ws.get(key)
    if ws is None:
        ws = _default_ws[key] = Workspace(device)
    return ws


def _stream_ptr(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SV_F32
    if t.dtype == torch.bfloat16:
        return SV_BF16
    raise TypeError(f"logits must be float32 or bfloat16, got {t.dtype}")


def _logits(t: torch.Tensor, ndim: int, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dim() != ndim:
        raise ValueError(f"{name} must be {ndim}-d, got shape {tuple(t.shape)}")
    if t.numel() > 0 and t.shape[-1] > 1 and t.stride(-1) != 1:
        raise ValueError(f"{name}: the vocabulary axis must be contiguous")
    return _dtype_code(t), t.stride()


def _tokens(t: torch.Tensor, shape, device, name: str) -> torch.Tensor:
    if not isinstance(t, torch.Tensor) or t.device != device or t.dtype != torch.int32:
        raise TypeError(f"{name} must be an int32 tensor on {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.contiguous()


def _out(out, key, shape, dtype, device):
    if out is not None and key in out:
        t = out[key]
        if tuple(t.shape) != tuple(shape) or t.dtype != dtype or not t.is_contiguous():
            raise ValueError(f"out[{key!r}] must be a contiguous {dtype} tensor {tuple(shape)}")
        return t
    return torch.empty(shape, dtype=dtype, device=device)


def stochastic(target: torch.Tensor, draft: torch.Tensor, draft_tokens: torch.Tensor,
               temperature: float, seed: int, seq_offset: int = 0, *, probs: bool = False,
               out: dict | None = None, workspace: Workspace | None = None,
               stream=None) -> dict:
    """Stochastic verify: target [B,k+1,V], draft [B,k,V], draft_tokens [B,k].

    Returns accepted_len [B], out_tokens [B,k+1] (and probs [B,k,2] when
    asked), all on the device; nothing is synchronised.
    """
    lib = load_library()
    tc, (tsb, tsp, _) = _logits(target, 3, "target")
    dc, (dsb, dsp, _) = _logits(draft, 3, "draft")
    B, kp1, V = target.shape
    k = kp1 - 1
    if tuple(draft.shape) != (B, k, V) or draft.device != target.device:
        raise ValueError("draft must be [B, k, V] on the target's device")
    dev = target.device
    tok = _tokens(draft_tokens, (B, k), dev, "draft_tokens")
    res = {"accepted_len": _out(out, "accepted_len", (B,), torch.int32, dev),
           "out_tokens": _out(out, "out_tokens", (B, k + 1), torch.int32, dev)}
    if probs:
        res["probs"] = _out(out, "probs", (B, k, 2), torch.float32, dev)
    ws = workspace or default_workspace(dev)
    ws.ensure(workspace_size(B, 1, k, V), stream)
    with torch.cuda.device(dev):
        code = lib.spec_verify_stochastic(
            target.data_ptr(), tc, tsb, tsp, draft.data_ptr(), dc, dsb, dsp, tok.data_ptr(),
            B, k, V, float(temperature), int(seed) & (2**64 - 1), int(seq_offset) & 0xFFFFFFFF,
            res["accepted_len"].data_ptr(), res["out_tokens"].data_ptr(),
            res["probs"].data_ptr() if probs else None, ws.buf.data_ptr(), ws.nbytes,
            _stream_ptr(stream, dev))
    _check(code, "spec_verify_stochastic")
    return res


def greedy(target: torch.Tensor, draft_tokens: torch.Tensor, *, out: dict | None = None,
           workspace: Workspace | None = None, stream=None) -> dict:
    """Greedy verify: target [B,k+1,V], draft_tokens [B,k]."""
    lib = load_library()
    tc, (tsb, tsp, _) = _logits(target, 3, "target")
    B, kp1, V = target.shape
    k = kp1 - 1
    dev = target.device
    tok = _tokens(draft_tokens, (B, k), dev, "draft_tokens")
    res = {"accepted_len": _out(out, "accepted_len", (B,), torch.int32, dev),
           "out_tokens": _out(out, "out_tokens", (B, k + 1), torch.int32, dev)}
    ws = workspace or default_workspace(dev)
    ws.ensure(workspace_size(B, 1, k, V), stream)
    with torch.cuda.device(dev):
        code = lib.spec_verify_greedy(
            target.data_ptr(), tc, tsb, tsp, tok.data_ptr(), B, k, V,
            res["accepted_len"].data_ptr(), res["out_tokens"].data_ptr(), ws.buf.data_ptr(),
            ws.nbytes, _stream_ptr(stream, dev))
    _check(code, "spec_verify_greedy")
    return res


def multi_candidate(target: torch.Tensor, cand_tokens: torch.Tensor, *, out: dict | None = None,
                    workspace: Workspace | None = None, stream=None) -> dict:
    """Multi-candidate verify: target [B,G,k+1,V], cand_tokens [B,G,k]."""
    lib = load_library()
    tc, (tsb, tsg, tsp, _) = _logits(target, 4, "target")
    B, G, kp1, V = target.shape
    k = kp1 - 1
    dev = target.device
    tok = _tokens(cand_tokens, (B, G, k), dev, "cand_tokens")
    res = {"best_candidate": _out(out, "best_candidate", (B,), torch.int32, dev),
           "accepted_len": _out(out, "accepted_len", (B,), torch.int32, dev),
           "out_tokens": _out(out, "out_tokens", (B, k + 1), torch.int32, dev)}
    ws = workspace or default_workspace(dev)
    ws.ensure(workspace_size(B, G, k, V), stream)
    with torch.cuda.device(dev):
        code = lib.spec_verify_multi_candidate(
            target.data_ptr(), tc, tsb, tsg, tsp, tok.data_ptr(), B, G, k, V,
            res["best_candidate"].data_ptr(), res["accepted_len"].data_ptr(),
            res["out_tokens"].data_ptr(), ws.buf.data_ptr(), ws.nbytes, _stream_ptr(stream, dev))
    _check(code, "spec_verify_multi_candidate")
    return res


def multi_candidate_rows(rows: torch.Tensor, row_of: torch.Tensor, cand_tokens: torch.Tensor, *,
                         out: dict | None = None, workspace: Workspace | None = None,
                         stream=None) -> dict:
    """Multi-candidate verify on deduplicated rows: rows [B,R,V], row_of
    [B,G,k+1] (int32, the row of each (b, g, i)), cand_tokens [B,G,k].  Same
    results as multi_candidate on rows gathered to [B,G,k+1,V]."""
    lib = load_library()
    tc, (tsb, tsr, _) = _logits(rows, 3, "rows")
    B, R, V = rows.shape
    if row_of.dim() != 3 or row_of.shape[0] != B:
        raise ValueError(f"row_of must be [B, G, k+1], got {tuple(row_of.shape)}")
    G, kp1 = int(row_of.shape[1]), int(row_of.shape[2])
    k = kp1 - 1
    dev = rows.device
    rmap = _tokens(row_of, (B, G, kp1), dev, "row_of")
    tok = _tokens(cand_tokens, (B, G, k), dev, "cand_tokens")
    res = {"best_candidate": _out(out, "best_candidate", (B,), torch.int32, dev),
           "accepted_len": _out(out, "accepted_len", (B,), torch.int32, dev),
           "out_tokens": _out(out, "out_tokens", (B, k + 1), torch.int32, dev)}
    ws = workspace or default_workspace(dev)
    ws.ensure(workspace_size(B, G, k, V), stream)
    with torch.cuda.device(dev):
        code = lib.spec_verify_multi_candidate_rows(
            rows.data_ptr(), tc, tsb, tsr, rmap.data_ptr(), tok.data_ptr(), B, G, k, R, V,
            res["best_candidate"].data_ptr(), res["accepted_len"].data_ptr(),
            res["out_tokens"].data_ptr(), ws.buf.data_ptr(), ws.nbytes, _stream_ptr(stream, dev))
    _check(code, "spec_verify_multi_candidate_rows")
    return res


def threshold(target: torch.Tensor, draft_tokens: torch.Tensor, temperature: float,
              threshold: float, *, out: dict | None = None, workspace: Workspace | None = None,
              stream=None) -> dict:
    """Threshold acceptance: target [B,k+1,V], draft_tokens [B,k]; accept the
    longest prefix whose probability under softmax(target/T) is at least
    `threshold`, then the argmax of the next row."""
    lib = load_library()
    tc, (tsb, tsp, _) = _logits(target, 3, "target")
    B, kp1, V = target.shape
    k = kp1 - 1
    dev = target.device
    tok = _tokens(draft_tokens, (B, k), dev, "draft_tokens")
    res = {"accepted_len": _out(out, "accepted_len", (B,), torch.int32, dev),
           "out_tokens": _out(out, "out_tokens", (B, k + 1), torch.int32, dev)}
    ws = workspace or default_workspace(dev)
    ws.ensure(workspace_size(B, 1, k, V), stream)
    with torch.cuda.device(dev):
        code = lib.spec_verify_threshold(
            target.data_ptr(), tc, tsb, tsp, tok.data_ptr(), B, k, V, float(temperature),
            float(threshold), res["accepted_len"].data_ptr(), res["out_tokens"].data_ptr(),
            ws.buf.data_ptr(), ws.nbytes, _stream_ptr(stream, dev))
    _check(code, "spec_verify_threshold")
    return res


def tree_workspace_size(B: int, N: int, V: int) -> int:
    return int(load_library().spec_verify_tree_workspace_size(B, N, V))


def tree_greedy(node_logits: torch.Tensor, parent: torch.Tensor, tokens: torch.Tensor, *,
                out: dict | None = None, workspace: Workspace | None = None,
                stream=None) -> dict:
    """Greedy verify of a draft token tree: node_logits [B,N,V] (row j = the
    target after the path to node j), parent [B,N] and tokens [B,N] int32.
    Returns accepted_len [B], path [B,N] and out_tokens [B,N]."""
    lib = load_library()
    tc, (tsb, tsn, _) = _logits(node_logits, 3, "node_logits")
    B, N, V = node_logits.shape
    dev = node_logits.device
    par = _tokens(parent, (B, N), dev, "parent")
    tok = _tokens(tokens, (B, N), dev, "tokens")
    res = {"accepted_len": _out(out, "accepted_len", (B,), torch.int32, dev),
           "path": _out(out, "path", (B, N), torch.int32, dev),
           "out_tokens": _out(out, "out_tokens", (B, N), torch.int32, dev)}
    ws = workspace or default_workspace(dev)
    ws.ensure(tree_workspace_size(B, N, V), stream)
    with torch.cuda.device(dev):
        code = lib.spec_verify_tree_greedy(
            node_logits.data_ptr(), tc, tsb, tsn, par.data_ptr(), tok.data_ptr(), B, N, V,
            res["accepted_len"].data_ptr(), res["path"].data_ptr(), res["out_tokens"].data_ptr(),
            ws.buf.data_ptr(), ws.nbytes, _stream_ptr(stream, dev))
    _check(code, "spec_verify_tree_greedy")
    return res


def tree_stochastic_workspace_size(B: int, N: int, V: int) -> int:
    return int(load_library().spec_verify_tree_stochastic_workspace_size(B, N, V))


def tree_stochastic(node_logits: torch.Tensor, parent: torch.Tensor, tokens: torch.Tensor,
                    temperature: float, seed: int, seq_offset: int = 0, *,
                    out: dict | None = None, workspace: Workspace | None = None,
                    stream=None) -> dict:
    """Stochastic verify of a draft token tree whose siblings are Top-K
    candidates: node_logits [B,N,V], parent [B,N] and tokens [B,N] int32 as
    for tree_greedy.  Returns accepted_len [B], path [B,N] and out_tokens
    [B,N] (the accepted tokens, the drawn token, then -1)."""
    lib = load_library()
    tc, (tsb, tsn, _) = _logits(node_logits, 3, "node_logits")
    B, N, V = node_logits.shape
    dev = node_logits.device
    par = _tokens(parent, (B, N), dev, "parent")
    tok = _tokens(tokens, (B, N), dev, "tokens")
    res = {"accepted_len": _out(out, "accepted_len", (B,), torch.int32, dev),
           "path": _out(out, "path", (B, N), torch.int32, dev),
           "out_tokens": _out(out, "out_tokens", (B, N), torch.int32, dev)}
    ws = workspace or default_workspace(dev)
    ws.ensure(tree_stochastic_workspace_size(B, N, V), stream)
    with torch.cuda.device(dev):
        code = lib.spec_verify_tree_stochastic(
            node_logits.data_ptr(), tc, tsb, tsn, par.data_ptr(), tok.data_ptr(), B, N, V,
            float(temperature), int(seed) & (2**64 - 1), int(seq_offset) & 0xFFFFFFFF,
            res["accepted_len"].data_ptr(), res["path"].data_ptr(), res["out_tokens"].data_ptr(),
            ws.buf.data_ptr(), ws.nbytes, _stream_ptr(stream, dev))
    _check(code, "spec_verify_tree_stochastic")
    return res


def commit(result: dict, seq_len: torch.Tensor, token_buf: torch.Tensor, *,
           next_input: torch.Tensor | None = None, workspace: Workspace | None = None,
           stream=None) -> None:
    """Device-side commit after a verify call: append each sequence's n + 1
    committed tokens (result["out_tokens"][b, :n+1], n = result["accepted_len"][b])
    to token_buf[b, seq_len[b]:], advance seq_len and write the next step's
    input token, all on the GPU (no host synchronisation).  token_buf is an
    int32 [B, capacity] tensor whose rows may be strided; tokens past capacity
    are dropped and flagged (SV_FLAG_CAPACITY) in `workspace` if given."""
    lib = load_library()
    acc, out = result["accepted_len"], result["out_tokens"]
    dev = acc.device
    B = int(acc.shape[0])
    k = int(out.shape[1]) - 1
    acc = _tokens(acc, (B,), dev, "accepted_len")
    out = _tokens(out, (B, k + 1), dev, "out_tokens")
    if (not isinstance(seq_len, torch.Tensor) or seq_len.dtype != torch.int32 or
            seq_len.device != dev or tuple(seq_len.shape) != (B,) or not seq_len.is_contiguous()):
        raise ValueError("seq_len must be a contiguous int32 [B] tensor on the verify device")
    if (token_buf.dtype != torch.int32 or token_buf.device != dev or token_buf.dim() != 2 or
            token_buf.shape[0] != B or (token_buf.shape[1] > 1 and token_buf.stride(1) != 1)):
        raise ValueError("token_buf must be an int32 [B, capacity] tensor with contiguous rows")
    if next_input is not None and (next_input.dtype != torch.int32 or next_input.device != dev or
                                   tuple(next_input.shape) != (B,) or
                                   not next_input.is_contiguous()):
        raise ValueError("next_input must be a contiguous int32 [B] tensor")
    cap = int(token_buf.shape[1])
    stride = int(token_buf.stride(0)) if B > 1 else cap
    with torch.cuda.device(dev):
        code = lib.spec_verify_commit(
            acc.data_ptr(), out.data_ptr(), B, k, seq_len.data_ptr(), token_buf.data_ptr(),
            max(stride, cap), cap, next_input.data_ptr() if next_input is not None else None,
            workspace.buf.data_ptr() if workspace is not None and workspace.buf is not None
            else None, _stream_ptr(stream, dev))
    _check(code, "spec_verify_commit")


def greedy_noalloc(target: torch.Tensor, draft_tokens: torch.Tensor, *,
                   out: dict | None = None, stream=None) -> dict:
    """Greedy verify that allocates no device memory inside the library.

    For callers that cannot allocate on the verify path (an external
    allocator or pool owns the device, or the call runs where an allocation
    may block or fail): the library uses its own fixed 2 MiB device array
    instead of a workspace.  Pass preallocated `out` tensors to keep this
    wrapper free of allocations as well.  Calls share that array, so order
    them on one stream; the first call on a device should come before any
    stream capture.
    """
    lib = load_library()
    tc, (tsb, tsp, _) = _logits(target, 3, "target")
    B, kp1, V = target.shape
    k = kp1 - 1
    dev = target.device
    tok = _tokens(draft_tokens, (B, k), dev, "draft_tokens")
    res = {"accepted_len": _out(out, "accepted_len", (B,), torch.int32, dev),
           "out_tokens": _out(out, "out_tokens", (B, k + 1), torch.int32, dev)}
    with torch.cuda.device(dev):
        code = lib.spec_verify_greedy_noalloc(
            target.data_ptr(), tc, tsb, tsp, tok.data_ptr(), B, k, V,
            res["accepted_len"].data_ptr(), res["out_tokens"].data_ptr(), _stream_ptr(stream, dev))
    _check(code, "spec_verify_greedy_noalloc")
    return res


def greedy_noalloc_device_status(clear: bool = True, device=None, stream=None) -> int:
    """Sticky SV_FLAG_* bits raised on the device by greedy_noalloc calls on
    `device` (synchronises the stream; allocates nothing)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else \
        torch.device(device)
    v = ctypes.c_uint32(0)
    with torch.cuda.device(dev):
        _check(load_library().spec_verify_greedy_noalloc_read_device_status(
            ctypes.byref(v), int(clear), _stream_ptr(stream, dev)),
            "spec_verify_greedy_noalloc_read_device_status")
    return int(v.value)


def philox4x32_10(counters: torch.Tensor, seed: int, stream=None) -> torch.Tensor:
    """Device Philox4x32-10 of each counter row ([n,4] int32 bit patterns)."""
    lib = load_library()
    if counters.dtype != torch.int32 or counters.dim() != 2 or counters.shape[1] != 4:
        raise TypeError("counters must be an int32 tensor [n, 4] (uint32 bit patterns)")
    c = counters.contiguous()
    out = torch.empty_like(c)
    with torch.cuda.device(c.device):
        code = lib.spec_verify_philox4x32_10(c.data_ptr(), c.shape[0], int(seed) & (2**64 - 1),
                                              out.data_ptr(), _stream_ptr(stream, c.device))
    _check(code, "spec_verify_philox4x32_10")
    return out
