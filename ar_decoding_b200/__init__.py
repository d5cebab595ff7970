"""Python binding of libtidar.so -- the GPU hot path of one TiDAR decode step.

Argument marshalling only: tensors are passed to the C ABI (include/tidar.h)
as raw device pointers with the current torch CUDA stream; every step of the
computation runs in the library's CUDA kernels.  There is no CPU fallback: if
libtidar.so is missing or a call fails, an exception is raised.

    out, lse = step_attn(q, k_blk, v_blk, cache, k, max_prefix_len=P)
    res = verify(logits, drafts, k, "greedy", block_guesses=g)
    released, n = commit(cache, res["accept_count"], k, max_prefix_len=P)
    reserve(cache, pool, k, max_prefix_len=P, returned=released, num_returned=n)

``cache`` is a mapping with the device tensors ``k_pages``/``v_pages``
[num_pages][Hkv][page][D], ``page_table`` [B][max_pages] int32 and
``seq_lens`` [B] int32 (the layout ``synth.make_cache`` produces).  ``pool``
maps ``free_pages`` [capacity] and ``free_count`` [1] (int32): the stack of free
page ids that ``reserve`` pops the next step's draft pages from, after pushing
the ids the commit released.
"""
from __future__ import annotations

import ctypes
import os
import re

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libtidar.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "tidar.h")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE = range(6)
F32, BF16 = 0, 1
GREEDY, REJECTION = 0, 1
PATH_AUTO, PATH_SIMT, PATH_TC05, PATH_DEC, PATH_PAIR = 0, 1, 2, 3, 4
DEVERR_BAD_PAGE, DEVERR_BAD_LEN, DEVERR_BAD_COUNT, DEVERR_TIMEOUT, DEVERR_LAYOUT = 1, 2, 4, 8, 16
DEVERR_POOL = 32
PART_STEP_KEYS, PART_APPEND = 1, 2
_PATHS = {"auto": PATH_AUTO, "simt": PATH_SIMT, "tc05": PATH_TC05, "dec": PATH_DEC,
          "pair": PATH_PAIR}


class TidarError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: status {status}")


class StepDesc(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("num_q_heads", ctypes.c_int32),
                ("num_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("k", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("max_prefix_len", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("softmax_scale", ctypes.c_float), ("path", ctypes.c_int32)]


class PagePool(ctypes.Structure):
    _fields_ = [("free_pages", ctypes.c_void_p), ("free_count", ctypes.c_void_p),
                ("capacity", ctypes.c_int32)]


class Sampling(ctypes.Structure):
    _fields_ = [("temperature", ctypes.c_float), ("top_p", ctypes.c_float)]


class KVCacheDesc(ctypes.Structure):
    _fields_ = [("k_pages", ctypes.c_void_p), ("v_pages", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("seq_lens", ctypes.c_void_p),
                ("num_pages", ctypes.c_int32), ("max_pages_per_seq", ctypes.c_int32)]


_lib = None


def lib():
    """The loaded libtidar.so (built in-tree by ``python -m ar_decoding_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "`python -m ar_decoding_b200.build` (needs nvcc)")
        L = ctypes.CDLL(LIB_PATH)
        P, S, I = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int32
        L.tidar_step_attn_workspace_bytes.argtypes = [P]
        L.tidar_step_attn_workspace_bytes.restype = S
        L.tidar_step_attn.argtypes = [P, P, P, P, P, P, P, P, S, P]
        L.tidar_step_attn.restype = ctypes.c_int
        L.tidar_step_attn_plan.argtypes = [P, P, P, P]
        L.tidar_step_attn_plan.restype = ctypes.c_int
        L.tidar_verify_workspace_bytes.argtypes = [I, I, I, ctypes.c_int]
        L.tidar_verify_workspace_bytes.restype = S
        L.tidar_verify.argtypes = [I, I, I, ctypes.c_int, ctypes.c_int, P, P, P, P, P, P, P, P, P, P,
                                   S, P]
        L.tidar_verify.restype = ctypes.c_int
        L.tidar_verify_noalloc.argtypes = [I, I, I, ctypes.c_int, ctypes.c_int, P, P, P, P, P, P, P,
                                           P, P, P]
        L.tidar_verify_noalloc.restype = ctypes.c_int
        L.tidar_verify_blockq.argtypes = [I, I, I, ctypes.c_int, P, P, P, P, P, P, P, P, P, P, P,
                                          S, P]
        L.tidar_verify_blockq.restype = ctypes.c_int
        L.tidar_commit.argtypes = [P, P, P, P, P, P]
        L.tidar_commit.restype = ctypes.c_int
        L.tidar_verify_commit.argtypes = [P, P, I, ctypes.c_int, ctypes.c_int, P, P, P, P, P, P, P, P, P, P, P,
                                          P, S, P]
        L.tidar_verify_commit.restype = ctypes.c_int
        L.tidar_reserve.argtypes = [P, P, P, P, P, P]
        L.tidar_reserve.restype = ctypes.c_int
        L.tidar_get_device_status.argtypes = [P, P]
        L.tidar_get_device_status.restype = ctypes.c_int
        L.tidar_status_string.argtypes = [ctypes.c_int]
        L.tidar_status_string.restype = ctypes.c_char_p
        L.tidar_last_cuda_error.argtypes = []
        L.tidar_last_cuda_error.restype = ctypes.c_char_p
        L.tidar_debug_set.argtypes = [ctypes.c_int, I]
        L.tidar_debug_set.restype = ctypes.c_int
        L.tidar_verify_sampled_workspace_bytes.argtypes = [I, I, I, ctypes.c_int]
        L.tidar_verify_sampled_workspace_bytes.restype = S
        L.tidar_verify_sampled.argtypes = [I, I, I, ctypes.c_int, ctypes.c_int, P, P, P, P, P, P, P,
                                           P, P, P, P, P, P, S, P]
        L.tidar_verify_sampled.restype = ctypes.c_int
        L.tidar_sample_drafts.argtypes = [I, I, I, ctypes.c_int, ctypes.c_int, P, P, P, P, P, P]
        L.tidar_sample_drafts.restype = ctypes.c_int
        L.tidar_step_attn_part.argtypes = [P, P, P, P, P, I, P, P, P, S, P]
        L.tidar_step_attn_part.restype = ctypes.c_int
        L.tidar_merge_attn.argtypes = [I, ctypes.c_int64, I, ctypes.c_int, P, P, P, P, P]
        L.tidar_merge_attn.restype = ctypes.c_int
        L.tidar_linear_workspace_bytes.argtypes = [I, I, I]
        L.tidar_linear_workspace_bytes.restype = S
        L.tidar_linear.argtypes = [I, I, I, ctypes.c_int, P, P, P, P, S, P]
        L.tidar_linear.restype = ctypes.c_int
        L.tidar_qkv_rope_workspace_bytes.argtypes = [P, I]
        L.tidar_qkv_rope_workspace_bytes.restype = S
        L.tidar_qkv_rope.argtypes = [P, I, P, P, P, ctypes.c_float, P, P, P, P, S, P]
        L.tidar_qkv_rope.restype = ctypes.c_int
        L.tidar_layer_step_workspace_bytes.argtypes = [P, I]
        L.tidar_layer_step_workspace_bytes.restype = S
        L.tidar_layer_step.argtypes = [P, P, I, P, P, P, ctypes.c_float, P, P, P, S, P]
        L.tidar_layer_step.restype = ctypes.c_int
        _lib = L
    return _lib


def header_functions() -> list[str]:
    """Names of the functions include/tidar.h declares."""
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[A-Za-z_][A-Za-z0-9_]*\s*\*?\s*(tidar_[a-z0-9_]+)\s*\(",
                                 text, flags=re.M)))


def _check(status: int, what: str):
    if status != OK:
        L = lib()
        msg = L.tidar_status_string(status).decode()
        if status == ERR_CUDA:
            msg += " (" + L.tidar_last_cuda_error().decode() + ")"
        raise TidarError(status, f"{what} failed: {msg}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_handle(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise ValueError(f"unsupported dtype {t.dtype}")


def _dev(t: torch.Tensor, name: str, dtype=None, device=None):
    """Every tensor handed to the library is a device pointer: a host tensor
    (or a strided view) is refused here rather than dereferenced on the GPU."""
    if not isinstance(t, torch.Tensor) or not t.is_cuda or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, the call's tensors are on {device}")


def _devopt(t, name: str, dtype=None, device=None):
    if t is not None:
        _dev(t, name, dtype, device)


def _check_verify_args(logits, drafts, draft_logits, uniforms, block_guesses, outputs, workspace):
    _dev(logits, "logits")
    dev = logits.device
    _devopt(drafts, "drafts", torch.int32, dev)
    _devopt(draft_logits, "draft_logits", logits.dtype, dev)
    _devopt(uniforms, "uniforms", torch.float32, dev)
    _devopt(block_guesses, "block_guesses", torch.int32, dev)
    _devopt(workspace, "workspace", None, dev)
    if outputs is not None:
        for key, t in outputs.items():
            _dev(t, key, torch.int32, dev)


def make_desc(q, k_blk, cache, k, max_prefix_len, scale=0.0, path="auto") -> StepDesc:
    B, R, Hq, D = q.shape
    return StepDesc(batch=B, num_q_heads=Hq, num_kv_heads=k_blk.shape[2], head_dim=D, k=k,
                    page_size=cache["k_pages"].shape[2], max_prefix_len=int(max_prefix_len),
                    dtype=_dtype_code(q), softmax_scale=float(scale), path=_PATHS[path])


def make_cache_desc(cache, device=None) -> KVCacheDesc:
    for n in ("k_pages", "v_pages", "page_table", "seq_lens"):
        _dev(cache[n], n, None, device)
    if cache["page_table"].dtype != torch.int32 or cache["seq_lens"].dtype != torch.int32:
        raise ValueError("page_table and seq_lens must be int32")
    return KVCacheDesc(k_pages=cache["k_pages"].data_ptr(), v_pages=cache["v_pages"].data_ptr(),
                       page_table=cache["page_table"].data_ptr(),
                       seq_lens=cache["seq_lens"].data_ptr(),
                       num_pages=cache["k_pages"].shape[0],
                       max_pages_per_seq=cache["page_table"].shape[1])


def plan(desc: StepDesc) -> tuple[int, int]:
    """(kernel family, KV splits) of the launch plan."""
    return plan_full(desc)[:2]


def plan_full(desc: StepDesc) -> tuple[int, int, int]:
    """(kernel family, KV splits, merge: 0 one split, 1 in the kernel, 2 a second launch)."""
    path, splits, merge = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    _check(lib().tidar_step_attn_plan(ctypes.byref(desc), ctypes.byref(path), ctypes.byref(splits),
                                      ctypes.byref(merge)), "tidar_step_attn_plan")
    return path.value, splits.value, merge.value


def step_attn_workspace_bytes(desc: StepDesc) -> int:
    return int(lib().tidar_step_attn_workspace_bytes(ctypes.byref(desc)))


def step_attn(q, k_blk, v_blk, cache, k, *, max_prefix_len, scale=0.0, path="auto", out=None,
              lse=None, want_lse=True, workspace=None, stream=None):
    """Three-zone step attention (+ draft-row K/V append).  Returns (out, lse)."""
    _dev(q, "q")
    dev = q.device
    _dev(k_blk, "k_blk", q.dtype, dev)
    _dev(v_blk, "v_blk", q.dtype, dev)
    desc = make_desc(q, k_blk, cache, k, max_prefix_len, scale, path)
    cdesc = make_cache_desc(cache, dev)
    if cache["k_pages"].dtype != q.dtype or cache["v_pages"].dtype != q.dtype:
        raise ValueError("the cache pages must have q's dtype")
    if out is None:
        out = torch.empty_like(q)
    if lse is None and want_lse:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    _dev(out, "out", q.dtype, dev)
    _devopt(lse, "lse", torch.float32, dev)
    need = step_attn_workspace_bytes(desc)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _devopt(workspace, "workspace", None, dev)
    wbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib().tidar_step_attn(ctypes.byref(desc), ctypes.byref(cdesc), _ptr(q), _ptr(k_blk),
                               _ptr(v_blk), _ptr(out), _ptr(lse), _ptr(workspace), wbytes,
                               _stream_handle(stream))
    _check(st, "tidar_step_attn")
    return out, lse


def _scratch(need, workspace, dev):
    """A workspace of at least `need` bytes on `dev` (allocated when None)."""
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _devopt(workspace, "workspace", None, dev)
    return workspace, (workspace.numel() * workspace.element_size() if workspace is not None else 0)


def linear_workspace_bytes(rows: int, out_features: int, in_features: int) -> int:
    return int(lib().tidar_linear_workspace_bytes(int(rows), int(out_features), int(in_features)))


def linear(x, w, *, out=None, workspace=None, stream=None):
    """y = x w^T (bf16; x [rows][in], w [out][in]) on the tensor cores."""
    _dev(x, "x", torch.bfloat16)
    _dev(w, "w", torch.bfloat16, x.device)
    N, K = w.shape
    if x.numel() % K:
        raise ValueError(f"x has {x.numel()} elements, not a whole number of rows of {K} features")
    rows = x.numel() // K
    if out is None:
        shape = (*x.shape[:-1], N) if x.shape[-1] == K else (rows, N)
        out = torch.empty(shape, dtype=torch.bfloat16, device=x.device)
    if out.numel() != rows * N:
        raise ValueError(f"out has {out.numel()} elements, expected {rows} x {N}")
    _dev(out, "out", torch.bfloat16, x.device)
    ws, wbytes = _scratch(linear_workspace_bytes(rows, N, K) if rows else 0, workspace, x.device)
    _check(lib().tidar_linear(rows, N, K, BF16, _ptr(x), _ptr(w), _ptr(out), _ptr(ws), wbytes,
                              _stream_handle(stream)), "tidar_linear")
    return out


def _layer_desc(x, k, Hq, Hkv, max_prefix_len, page_size=64, path="auto"):
    B, R, _ = x.shape
    if R != (1 if k == 0 else k + k * k):
        raise ValueError(f"x has {R} rows per sequence, k = {k} needs {1 if k == 0 else k + k * k}")
    return StepDesc(batch=B, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=128, k=k,
                    page_size=page_size, max_prefix_len=int(max_prefix_len), dtype=BF16,
                    softmax_scale=0.0, path=_PATHS[path])


def qkv_rope(x, w_qkv, seq_lens, k, num_q_heads, num_kv_heads, *, max_prefix_len,
             rope_base=10000.0, out=None, workspace=None, stream=None):
    """Query/key/value projection of the step rows x [B][R][d_model] with the
    rotary embedding at their zone positions.  Returns (q, k_blk, v_blk)."""
    _dev(x, "x", torch.bfloat16)
    dev = x.device
    _dev(w_qkv, "w_qkv", torch.bfloat16, dev)
    _dev(seq_lens, "seq_lens", torch.int32, dev)
    B, R, dm = x.shape
    Hq, Hkv = num_q_heads, num_kv_heads
    if tuple(w_qkv.shape) != ((Hq + 2 * Hkv) * 128, dm):
        raise ValueError(f"w_qkv is {tuple(w_qkv.shape)}, expected {((Hq + 2 * Hkv) * 128, dm)}")
    desc = _layer_desc(x, k, Hq, Hkv, max_prefix_len)
    if out is None:
        out = (torch.empty((B, R, Hq, 128), dtype=torch.bfloat16, device=dev),
               torch.empty((B, R, Hkv, 128), dtype=torch.bfloat16, device=dev),
               torch.empty((B, R, Hkv, 128), dtype=torch.bfloat16, device=dev))
    for name, t in zip(("q", "k_blk", "v_blk"), out):
        _dev(t, name, torch.bfloat16, dev)
    q, kb, vb = out
    ws, wbytes = _scratch(int(lib().tidar_qkv_rope_workspace_bytes(ctypes.byref(desc), dm)), workspace, dev)
    _check(lib().tidar_qkv_rope(ctypes.byref(desc), dm, _ptr(x), _ptr(w_qkv), _ptr(seq_lens),
                                float(rope_base), _ptr(q), _ptr(kb), _ptr(vb), _ptr(ws), wbytes,
                                _stream_handle(stream)), "tidar_qkv_rope")
    return q, kb, vb


def layer_step_workspace_bytes(desc: StepDesc, d_model: int) -> int:
    return int(lib().tidar_layer_step_workspace_bytes(ctypes.byref(desc), int(d_model)))


def layer_step(x, w_qkv, w_o, cache, k, num_q_heads, num_kv_heads, *, max_prefix_len,
               rope_base=10000.0, path="auto", out=None, lse=None, want_lse=True,
               workspace=None, stream=None):
    """One layer of a TiDAR step: projection + rotary embedding, three-zone
    step attention (with the draft-row append), output projection.
    Returns (y [B][R][d_model], lse [B][R][Hq])."""
    _dev(x, "x", torch.bfloat16)
    dev = x.device
    _dev(w_qkv, "w_qkv", torch.bfloat16, dev)
    _dev(w_o, "w_o", torch.bfloat16, dev)
    B, R, dm = x.shape
    desc = _layer_desc(x, k, num_q_heads, num_kv_heads, max_prefix_len,
                       page_size=cache["k_pages"].shape[2], path=path)
    cdesc = make_cache_desc(cache, dev)
    if out is None:
        out = torch.empty((B, R, dm), dtype=torch.bfloat16, device=dev)
    if lse is None and want_lse:
        lse = torch.empty((B, R, num_q_heads), dtype=torch.float32, device=dev)
    _dev(out, "out", torch.bfloat16, dev)
    _devopt(lse, "lse", torch.float32, dev)
    need = layer_step_workspace_bytes(desc, dm)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _dev(workspace, "workspace", None, dev)
    st = lib().tidar_layer_step(ctypes.byref(desc), ctypes.byref(cdesc), dm, _ptr(x), _ptr(w_qkv),
                                _ptr(w_o), float(rope_base), _ptr(out), _ptr(lse), _ptr(workspace),
                                workspace.numel(), _stream_handle(stream))
    _check(st, "tidar_layer_step")
    return out, lse


def step_attn_part(q, k_blk, v_blk, cache, k, flags, *, max_prefix_len, scale=0.0, path="auto",
                   out=None, lse=None, workspace=None, stream=None):
    """Step attention over one slice of a sequence's prefix (context
    parallelism): flags PART_STEP_KEYS also attends the step keys,
    PART_APPEND writes the draft rows.  Returns (out, lse)."""
    _dev(q, "q")
    dev = q.device
    _dev(k_blk, "k_blk", q.dtype, dev)
    _dev(v_blk, "v_blk", q.dtype, dev)
    desc = make_desc(q, k_blk, cache, k, max_prefix_len, scale, path)
    cdesc = make_cache_desc(cache, dev)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(q.shape[:3], dtype=torch.float32, device=dev)
    _dev(out, "out", q.dtype, dev)
    _dev(lse, "lse", torch.float32, dev)
    need = step_attn_workspace_bytes(desc)
    if workspace is None and need:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _devopt(workspace, "workspace", None, dev)
    wbytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    st = lib().tidar_step_attn_part(ctypes.byref(desc), ctypes.byref(cdesc), _ptr(q), _ptr(k_blk),
                                    _ptr(v_blk), int(flags), _ptr(out), _ptr(lse), _ptr(workspace),
                                    wbytes, _stream_handle(stream))
    _check(st, "tidar_step_attn_part")
    return out, lse


def merge_attn(parts_out, parts_lse, *, out=None, lse=None, stream=None):
    """Log-sum-exp merge of attention results over disjoint key sets:
    parts_out [nparts][...][D], parts_lse [nparts][...] -> (out, lse)."""
    _dev(parts_out, "parts_out")
    dev = parts_out.device
    _dev(parts_lse, "parts_lse", torch.float32, dev)
    nparts, D = parts_out.shape[0], parts_out.shape[-1]
    rows = parts_lse[0].numel()
    if tuple(parts_out.shape[:-1]) != tuple(parts_lse.shape):
        raise ValueError("parts_out and parts_lse disagree in shape")
    if out is None:
        out = torch.empty(parts_out.shape[1:], dtype=parts_out.dtype, device=dev)
    if lse is None:
        lse = torch.empty(parts_lse.shape[1:], dtype=torch.float32, device=dev)
    _dev(out, "out", parts_out.dtype, dev)
    _dev(lse, "lse", torch.float32, dev)
    st = lib().tidar_merge_attn(nparts, rows, D, _dtype_code(parts_out), _ptr(parts_out),
                                _ptr(parts_lse), _ptr(out), _ptr(lse), _stream_handle(stream))
    _check(st, "tidar_merge_attn")
    return out, lse


def verify_workspace_bytes(B, k, V, mode) -> int:
    return int(lib().tidar_verify_workspace_bytes(B, k, V, mode))


def verify(logits, drafts, k, mode="greedy", *, draft_logits=None, uniforms=None,
           block_guesses=None, outputs=None, workspace=None, stream=None):
    """Verification, acceptance and block selection.  Returns a dict of device tensors:
    accept_count [B], out_tokens [B][n], next_drafts [B][k], selected_block [B]."""
    m = mode if isinstance(mode, int) else {"greedy": GREEDY, "rejection": REJECTION}[mode]
    _dev(logits, "logits")
    B, n, V = logits.shape
    dev = logits.device
    if outputs is None:
        outputs = dict(accept_count=torch.empty(B, dtype=torch.int32, device=dev),
                       out_tokens=torch.empty((B, n), dtype=torch.int32, device=dev),
                       next_drafts=torch.empty((B, max(k, 1)), dtype=torch.int32, device=dev),
                       selected_block=torch.empty(B, dtype=torch.int32, device=dev))
    need = verify_workspace_bytes(B, k, V, m)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check_verify_args(logits, drafts, draft_logits, uniforms, block_guesses, outputs, workspace)
    st = lib().tidar_verify(B, k, V, _dtype_code(logits), m, _ptr(logits), _ptr(drafts),
                            _ptr(draft_logits), _ptr(uniforms), _ptr(block_guesses),
                            _ptr(outputs["accept_count"]), _ptr(outputs["out_tokens"]),
                            _ptr(outputs["next_drafts"]) if k > 0 else None,
                            _ptr(outputs["selected_block"]), _ptr(workspace),
                            workspace.numel(), _stream_handle(stream))
    _check(st, "tidar_verify")
    return outputs


def verify_blockq(logits, drafts, k, prev_block_logits, draft_block, uniforms, *,
                  block_guesses=None, outputs=None, workspace=None, stream=None):
    """Rejection verification with q read in place from the previous step's mask
    blocks: prev_block_logits [B][k][k][V], draft_block [B] int32 (last step's
    selected_block).  Returns the same dict as ``verify``."""
    _dev(logits, "logits")
    B, n, V = logits.shape
    dev = logits.device
    if outputs is None:
        outputs = dict(accept_count=torch.empty(B, dtype=torch.int32, device=dev),
                       out_tokens=torch.empty((B, n), dtype=torch.int32, device=dev),
                       next_drafts=torch.empty((B, max(k, 1)), dtype=torch.int32, device=dev),
                       selected_block=torch.empty(B, dtype=torch.int32, device=dev))
    need = verify_workspace_bytes(B, k, V, REJECTION)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check_verify_args(logits, drafts, prev_block_logits, uniforms, block_guesses, outputs,
                       workspace)
    _devopt(draft_block, "draft_block", torch.int32, dev)
    st = lib().tidar_verify_blockq(B, k, V, _dtype_code(logits), _ptr(logits), _ptr(drafts),
                                   _ptr(prev_block_logits), _ptr(draft_block), _ptr(uniforms),
                                   _ptr(block_guesses), _ptr(outputs["accept_count"]),
                                   _ptr(outputs["out_tokens"]),
                                   _ptr(outputs["next_drafts"]) if k > 0 else None,
                                   _ptr(outputs["selected_block"]), _ptr(workspace),
                                   workspace.numel(), _stream_handle(stream))
    _check(st, "tidar_verify_blockq")
    return outputs


def verify_sampled(logits, drafts, k, mode="rejection", *, temperature=1.0, top_p=1.0,
                   draft_logits=None, prev_block_logits=None, draft_block=None, uniforms=None,
                   block_guesses=None, outputs=None, workspace=None, stream=None):
    """Verification with the sampling transform (temperature, nucleus top_p)
    applied to p and q.  q comes from draft_logits [B][k-1][V] or, with
    prev_block_logits [B][k][k][V] and draft_block [B], in place from the
    previous step's mask blocks.  Returns the same dict as ``verify``."""
    m = mode if isinstance(mode, int) else {"greedy": GREEDY, "rejection": REJECTION}[mode]
    _dev(logits, "logits")
    B, n, V = logits.shape
    dev = logits.device
    if outputs is None:
        outputs = dict(accept_count=torch.empty(B, dtype=torch.int32, device=dev),
                       out_tokens=torch.empty((B, n), dtype=torch.int32, device=dev),
                       next_drafts=torch.empty((B, max(k, 1)), dtype=torch.int32, device=dev),
                       selected_block=torch.empty(B, dtype=torch.int32, device=dev))
    need = int(lib().tidar_verify_sampled_workspace_bytes(B, k, V, m))
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check_verify_args(logits, drafts, draft_logits, uniforms, block_guesses, outputs, workspace)
    _devopt(prev_block_logits, "prev_block_logits", logits.dtype, dev)
    _devopt(draft_block, "draft_block", torch.int32, dev)
    sp = Sampling(temperature=float(temperature), top_p=float(top_p))
    st = lib().tidar_verify_sampled(B, k, V, _dtype_code(logits), m, ctypes.byref(sp), _ptr(logits),
                                    _ptr(drafts), _ptr(draft_logits), _ptr(prev_block_logits),
                                    _ptr(draft_block), _ptr(uniforms), _ptr(block_guesses),
                                    _ptr(outputs["accept_count"]), _ptr(outputs["out_tokens"]),
                                    _ptr(outputs["next_drafts"]) if k > 0 else None,
                                    _ptr(outputs["selected_block"]), _ptr(workspace),
                                    workspace.numel(), _stream_handle(stream))
    _check(st, "tidar_verify_sampled")
    return outputs


def sample_drafts(block_logits, selected_block, k, mode="rejection", *, temperature=1.0, top_p=1.0,
                  uniforms=None, next_drafts=None, stream=None):
    """The next drafts from slots 2..k of each sequence's selected mask block
    (block_logits [B][k][k][V], selected_block [B] int32); writes entries
    1..k-1 of next_drafts [B][k] (entry 0, t*, is left alone).  Returns it."""
    m = mode if isinstance(mode, int) else {"greedy": GREEDY, "rejection": REJECTION}[mode]
    _dev(block_logits, "block_logits")
    dev = block_logits.device
    B, kk, k2, V = block_logits.shape
    if kk != k or k2 != k:
        raise ValueError(f"block_logits is {tuple(block_logits.shape)}, k = {k}")
    _dev(selected_block, "selected_block", torch.int32, dev)
    _devopt(uniforms, "uniforms", torch.float32, dev)
    if next_drafts is None:
        next_drafts = torch.full((B, max(k, 1)), -1, dtype=torch.int32, device=dev)
    _dev(next_drafts, "next_drafts", torch.int32, dev)
    sp = Sampling(temperature=float(temperature), top_p=float(top_p))
    st = lib().tidar_sample_drafts(B, k, V, _dtype_code(block_logits), m, ctypes.byref(sp),
                                   _ptr(block_logits), _ptr(selected_block), _ptr(uniforms),
                                   _ptr(next_drafts), _stream_handle(stream))
    _check(st, "tidar_sample_drafts")
    return next_drafts


VERIFY_NOALLOC_MAX_SCRATCH_BYTES = 4 << 20


def verify_noalloc(logits, drafts, k, mode="greedy", *, draft_logits=None, uniforms=None,
                   block_guesses=None, outputs=None, stream=None):
    """tidar_verify without a workspace: the library's fixed device scratch is used
    (for callers that cannot allocate at this point, e.g. inside graph capture
    once the first call on the device has been made outside it)."""
    m = mode if isinstance(mode, int) else {"greedy": GREEDY, "rejection": REJECTION}[mode]
    _dev(logits, "logits")
    B, n, V = logits.shape
    dev = logits.device
    if outputs is None:
        outputs = dict(accept_count=torch.empty(B, dtype=torch.int32, device=dev),
                       out_tokens=torch.empty((B, n), dtype=torch.int32, device=dev),
                       next_drafts=torch.empty((B, max(k, 1)), dtype=torch.int32, device=dev),
                       selected_block=torch.empty(B, dtype=torch.int32, device=dev))
    _check_verify_args(logits, drafts, draft_logits, uniforms, block_guesses, outputs, None)
    st = lib().tidar_verify_noalloc(B, k, V, _dtype_code(logits), m, _ptr(logits), _ptr(drafts),
                                    _ptr(draft_logits), _ptr(uniforms), _ptr(block_guesses),
                                    _ptr(outputs["accept_count"]), _ptr(outputs["out_tokens"]),
                                    _ptr(outputs["next_drafts"]) if k > 0 else None,
                                    _ptr(outputs["selected_block"]), _stream_handle(stream))
    _check(st, "tidar_verify_noalloc")
    return outputs


def commit(cache, accept_count, k, *, max_prefix_len, head_dim=None, num_q_heads=None,
           released=None, num_released=None, stream=None):
    """KV commit/evict in place.  Returns (released [B*(ceil(n/ps)+1)], num_released [1])."""
    kp = cache["k_pages"]
    B = cache["seq_lens"].shape[0]
    Hkv, ps, D = kp.shape[1], kp.shape[2], kp.shape[3]
    n = max(k, 1)
    desc = StepDesc(batch=B, num_q_heads=num_q_heads or Hkv, num_kv_heads=Hkv, head_dim=D, k=k,
                    page_size=ps, max_prefix_len=int(max_prefix_len), dtype=_dtype_code(kp),
                    softmax_scale=0.0, path=PATH_AUTO)
    cdesc = make_cache_desc(cache, kp.device)
    cap = B * ((n + ps - 1) // ps + 1)
    if released is None:
        released = torch.empty(cap, dtype=torch.int32, device=kp.device)
    if num_released is None:
        num_released = torch.empty(1, dtype=torch.int32, device=kp.device)
    _dev(accept_count, "accept_count", torch.int32, kp.device)
    _dev(released, "released", torch.int32, kp.device)
    _dev(num_released, "num_released", torch.int32, kp.device)
    st = lib().tidar_commit(ctypes.byref(desc), ctypes.byref(cdesc), _ptr(accept_count),
                            _ptr(released), _ptr(num_released), _stream_handle(stream))
    _check(st, "tidar_commit")
    return released, num_released


def verify_commit(logits, drafts, cache, k, mode="greedy", *, max_prefix_len, draft_logits=None,
                  uniforms=None, block_guesses=None, outputs=None, released=None, num_released=None,
                  workspace=None, stream=None):
    """``verify`` then ``commit`` on its accept counts, as one call (greedy:
    two launches).  Returns (outputs dict as ``verify``, released, num_released)."""
    m = mode if isinstance(mode, int) else {"greedy": GREEDY, "rejection": REJECTION}[mode]
    _dev(logits, "logits")
    B, n, V = logits.shape
    dev = logits.device
    kp = cache["k_pages"]
    if cache["seq_lens"].shape[0] != B:
        raise ValueError(f"the cache holds {cache['seq_lens'].shape[0]} sequences, the logits {B}")
    Hkv, ps, D = kp.shape[1], kp.shape[2], kp.shape[3]
    desc = StepDesc(batch=B, num_q_heads=Hkv, num_kv_heads=Hkv, head_dim=D, k=k, page_size=ps,
                    max_prefix_len=int(max_prefix_len), dtype=_dtype_code(kp), softmax_scale=0.0,
                    path=PATH_AUTO)
    cdesc = make_cache_desc(cache, dev)
    if outputs is None:
        outputs = dict(accept_count=torch.empty(B, dtype=torch.int32, device=dev),
                       out_tokens=torch.empty((B, n), dtype=torch.int32, device=dev),
                       next_drafts=torch.empty((B, max(k, 1)), dtype=torch.int32, device=dev),
                       selected_block=torch.empty(B, dtype=torch.int32, device=dev))
    cap = B * ((max(k, 1) + ps - 1) // ps + 1)
    if released is None:
        released = torch.empty(cap, dtype=torch.int32, device=dev)
    if num_released is None:
        num_released = torch.empty(1, dtype=torch.int32, device=dev)
    _dev(released, "released", torch.int32, dev)
    _dev(num_released, "num_released", torch.int32, dev)
    need = verify_workspace_bytes(B, k, V, m)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=dev)
    _check_verify_args(logits, drafts, draft_logits, uniforms, block_guesses, outputs, workspace)
    st = lib().tidar_verify_commit(ctypes.byref(desc), ctypes.byref(cdesc), V, _dtype_code(logits), m,
                                   _ptr(logits), _ptr(drafts), _ptr(draft_logits), _ptr(uniforms),
                                   _ptr(block_guesses), _ptr(outputs["accept_count"]),
                                   _ptr(outputs["out_tokens"]),
                                   _ptr(outputs["next_drafts"]) if k > 0 else None,
                                   _ptr(outputs["selected_block"]), _ptr(released), _ptr(num_released),
                                   _ptr(workspace), workspace.numel(), _stream_handle(stream))
    _check(st, "tidar_verify_commit")
    return outputs, released, num_released


def reserve(cache, pool, k, *, max_prefix_len, returned=None, num_returned=None, stream=None):
    """Pages for the draft rows of the next step, popped from a device stack.

    ``pool`` maps ``free_pages`` [capacity] int32 (ids [0, free_count) free)
    and ``free_count`` [1] int32, both device tensors.  ``returned`` /
    ``num_returned`` (e.g. what ``commit`` returned) are pushed first.
    Updates ``cache["page_table"]`` and the pool in place."""
    kp = cache["k_pages"]
    B = cache["seq_lens"].shape[0]
    Hkv, ps, D = kp.shape[1], kp.shape[2], kp.shape[3]
    desc = StepDesc(batch=B, num_q_heads=Hkv, num_kv_heads=Hkv, head_dim=D, k=k, page_size=ps,
                    max_prefix_len=int(max_prefix_len), dtype=_dtype_code(kp), softmax_scale=0.0,
                    path=PATH_AUTO)
    cdesc = make_cache_desc(cache, kp.device)
    fp, fc = pool["free_pages"], pool["free_count"]
    _dev(fc, "free_count", torch.int32, kp.device)
    if fp.numel():
        _dev(fp, "free_pages", torch.int32, kp.device)
    elif fp.dtype != torch.int32:
        raise ValueError("free_pages must be int32")
    _devopt(returned, "returned", torch.int32, kp.device)
    _devopt(num_returned, "num_returned", torch.int32, kp.device)
    p = PagePool(free_pages=fp.data_ptr() if fp.numel() else None, free_count=fc.data_ptr(),
                 capacity=int(fp.numel()))
    st = lib().tidar_reserve(ctypes.byref(desc), ctypes.byref(cdesc), ctypes.byref(p),
                             _ptr(returned), _ptr(num_returned), _stream_handle(stream))
    _check(st, "tidar_reserve")


DEBUG_STARVE_ATTENTION_LOADS, DEBUG_FORCE_SPLIT_PARTIALS = 1, 2


def debug_set(knob: int, value: int) -> None:
    """Test hooks (include/tidar.h): DEBUG_STARVE_ATTENTION_LOADS makes the
    tensor-core attention's bounded waits run out; DEBUG_FORCE_SPLIT_PARTIALS
    sends key splits through workspace partials instead of the on-chip merge."""
    _check(lib().tidar_debug_set(knob, int(value)), "tidar_debug_set")


def device_status(stream=None) -> tuple[int, int]:
    """Synchronises the stream; returns (status, error bits) and clears the word."""
    bits = ctypes.c_uint32()
    st = lib().tidar_get_device_status(_stream_handle(stream), ctypes.byref(bits))
    return st, bits.value
