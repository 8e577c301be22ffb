"""Thin ctypes binding of libuno (include/uno.h).

Argument marshalling only: every step of the decode iteration runs in the
library's CUDA kernels.  PyTorch tensors are accepted where the C ABI takes
device or host pointers; PyTorch provides device memory and streams, nothing
else.  When the shared library is missing, loading raises: there is no
fallback path.
"""

import ctypes
import os
import re

PKG = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(PKG)
LIB_PATH = os.path.join(PKG, "libuno.so")
HEADER = os.path.join(ROOT, "include", "uno.h")

UNO_F32, UNO_BF16 = 0, 1
UNO_OK, UNO_ERR_ARG, UNO_ERR_OOM, UNO_ERR_CAPACITY, UNO_ERR_CUDA, UNO_ERR_DEVICE_CHECK, \
    UNO_ERR_UNSUPPORTED = range(7)
UNO_DBG_LOGITS_DRAFT, UNO_DBG_LOGITS_VERIFY, UNO_DBG_DRAFTS, UNO_DBG_LOGITS_AR, \
    UNO_DBG_TOPP_DRAFT, UNO_DBG_TOPP_VERIFY, UNO_DBG_COHORT_LOGITS, UNO_DBG_COHORT_DRAFTS, \
    UNO_DBG_TREE_CHAINS, UNO_DBG_TREE_LOGITS, UNO_DBG_TREE_WALK = range(11)
PROJ = ("q", "k", "v", "o", "gate", "up", "down")
N_PROJ = len(PROJ)

_ERR_NAMES = {0: "UNO_OK", 1: "UNO_ERR_ARG", 2: "UNO_ERR_OOM", 3: "UNO_ERR_CAPACITY",
              4: "UNO_ERR_CUDA", 5: "UNO_ERR_DEVICE_CHECK", 6: "UNO_ERR_UNSUPPORTED"}


class UnoError(RuntimeError):
    def __init__(self, code, msg=""):
        super().__init__(f"{_ERR_NAMES.get(code, code)}: {msg}")
        self.code = code


class UnoShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("n_layers", "d_model", "n_heads", "n_kv_heads", "head_dim", "ffn_dim", "vocab",
                 "mask_id")] + \
               [("rope_theta", ctypes.c_float), ("rms_eps", ctypes.c_float),
                ("temperature", ctypes.c_float), ("dtype", ctypes.c_int32)]


_PP = ctypes.POINTER(ctypes.c_void_p)


class UnoWeights(ctypes.Structure):
    _fields_ = [("embed", ctypes.c_void_p), ("lm_head", ctypes.c_void_p),
                ("final_norm", ctypes.c_void_p), ("attn_norm", _PP), ("ffn_norm", _PP),
                ("w", _PP * N_PROJ), ("lora_A", _PP * N_PROJ), ("lora_B", _PP * N_PROJ)]


_lib = None


def load_library(path=LIB_PATH):
    """Load libuno.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"libuno.so not found at {path}: build it with "
                           "`python -m lossless_diffusion_draft_b200.build`")
    lib = ctypes.CDLL(path)
    i32, vp, u64, f32 = ctypes.c_int, ctypes.c_void_p, ctypes.c_uint64, ctypes.c_float
    sz = ctypes.c_size_t
    sig = {
        "uno_init": (i32, [ctypes.POINTER(UnoShape), ctypes.POINTER(UnoWeights), i32, f32, i32, i32,
                           i32, u64, vp, ctypes.POINTER(vp)]),
        "uno_prefill": (i32, [vp, i32, vp, i32, vp, vp, vp]),
        "uno_spec_step": (i32, [vp, i32, vp, vp, vp]),
        "uno_train_forward": (i32, [vp, i32, vp, i32, vp]),
        "uno_spec_step_cohorts": (i32, [vp, i32, vp, i32, vp, vp, vp]),
        "uno_ar_step": (i32, [vp, i32, vp, vp]),
        "uno_release": (i32, [vp, i32]),
        "uno_destroy": (i32, [vp]),
        "uno_last_error": (ctypes.c_char_p, [vp]),
        "uno_status": (i32, [vp]),
        "uno_request_state": (i32, [vp, i32, vp, vp]),
        "uno_debug_read": (i32, [vp, i32, vp, sz]),
        "uno_debug_kv": (i32, [vp, i32, i32, i32, i32, vp, vp]),
        "uno_gated_lora_linear_workspace_bytes": (sz, [i32, i32, i32, i32, i32]),
        "uno_gated_lora_linear": (i32, [i32, vp, vp, vp, vp, vp, i32, i32, i32, i32, f32, vp, vp,
                                        sz, vp]),
        "uno_debug_launch_counts": (i32, [vp]),
        "uno_set_graphs": (i32, [vp, i32]),
        "uno_set_pdl": (i32, [vp, i32]),
        "uno_set_fused": (i32, [vp, i32]),
        "uno_set_verify_split": (i32, [vp, i32]),
        "uno_set_counter_sync": (i32, [vp, i32]),
        "uno_debug_set_fixed_accept": (i32, [vp, i32]),
        "uno_set_top_p": (i32, [vp, f32]),
        "uno_set_tree": (i32, [vp, i32]),
        "uno_top_p_filter": (i32, [vp, i32, i32, f32, vp, vp]),
        "uno_debug_set_dep_wait": (i32, [vp, u64, ctypes.c_uint32]),
        "uno_profile_records": (i32, [vp, vp, i32]),
        "uno_profile_begin": (i32, [vp, ctypes.c_uint]),
        "uno_profile_end": (i32, [vp, vp, vp, vp]),
        "uno_spec_verify_workspace_bytes": (sz, [i32, i32, i32]),
        "uno_spec_verify": (i32, [vp, vp, vp, i32, i32, i32, u64, vp, vp, vp, vp, vp, sz, vp]),
        "uno_spec_verify_noalloc_max_bytes": (sz, []),
        "uno_spec_verify_noalloc": (i32, [vp, vp, vp, i32, i32, i32, u64, vp, vp, vp, vp, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def header_functions(header=HEADER):
    """Names of the functions include/uno.h declares."""
    text = open(header).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(uno_[a-z_0-9]+)\s*\(", text)))


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _check(code, ctx=None):
    if code != UNO_OK:
        msg = ""
        if ctx is not None:
            m = load_library().uno_last_error(ctx)
            msg = m.decode() if m else ""
        raise UnoError(code, msg)


def _stream_ptr(stream):
    if stream is None:
        return None
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


class Context:
    """An initialised uno_ctx plus the weight tensors it borrows."""

    def __init__(self, handle, shape, block_B, max_batch, keep):
        self.handle = handle
        self.shape = shape
        self.B = block_B
        self.max_batch = max_batch
        self._keep = keep

    def close(self):
        if self.handle:
            _check(load_library().uno_destroy(self.handle))
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


def uno_init(shape, params, lora_rank, lora_alpha, block_B, max_batch, max_ctx, seed, stream=None):
    """shape: dict (model shape + dtype "f32"/"bf16"); params: name -> device tensor."""
    lib = load_library()
    s = UnoShape(shape["n_layers"], shape["d_model"], shape["n_heads"], shape["n_kv_heads"],
                 shape["head_dim"], shape["ffn_dim"], shape["vocab"], shape["mask_id"],
                 shape["rope_theta"], shape["rms_eps"], shape.get("temperature", 1.0),
                 UNO_BF16 if shape["dtype"] == "bf16" else UNO_F32)
    L = shape["n_layers"]

    def arr(names):
        a = (ctypes.c_void_p * L)(*[params[n].data_ptr() for n in names])
        return a

    keep = []
    w = UnoWeights()
    w.embed = params["embed"].data_ptr()
    w.lm_head = params["lm_head"].data_ptr()
    w.final_norm = params["final_norm"].data_ptr()
    an = arr([f"l{l}.attn_norm" for l in range(L)])
    fn = arr([f"l{l}.ffn_norm" for l in range(L)])
    keep += [an, fn]
    w.attn_norm = ctypes.cast(an, _PP)
    w.ffn_norm = ctypes.cast(fn, _PP)
    for i, p in enumerate(PROJ):
        a = arr([f"l{l}.w_{p}" for l in range(L)])
        la = arr([f"l{l}.lora_{p}.A" for l in range(L)])
        lb = arr([f"l{l}.lora_{p}.B" for l in range(L)])
        keep += [a, la, lb]
        w.w[i] = ctypes.cast(a, _PP)
        w.lora_A[i] = ctypes.cast(la, _PP)
        w.lora_B[i] = ctypes.cast(lb, _PP)
    out = ctypes.c_void_p()
    code = lib.uno_init(ctypes.byref(s), ctypes.byref(w), lora_rank, lora_alpha, block_B, max_batch,
                        max_ctx, seed, _stream_ptr(stream), ctypes.byref(out))
    _check(code)
    return Context(out.value, shape, block_B, max_batch, [params] + keep)


def uno_prefill(ctx, prompts_dev, prompt_lens, streams=None):
    """prompts_dev: int32 CUDA tensor [n, stride]; returns the request ids."""
    lib = load_library()
    n = prompts_dev.shape[0]
    lens = (ctypes.c_int32 * n)(*[int(x) for x in prompt_lens])
    sids = None if streams is None else (ctypes.c_uint32 * n)(*[int(x) for x in streams])
    ids = (ctypes.c_int32 * n)()
    code = lib.uno_prefill(ctx.handle, n, _ptr(prompts_dev), prompts_dev.shape[1], lens, sids, ids)
    _check(code, ctx.handle)
    return list(ids)


def uno_train_forward(ctx, tokens_dev, logits_dev):
    """tokens_dev int32 CUDA [n_seq, 2L] (x then z) -> logits_dev f32 CUDA [n_seq, 2L, vocab]."""
    n_seq, two_l = tokens_dev.shape
    code = load_library().uno_train_forward(ctx.handle, n_seq, _ptr(tokens_dev), two_l // 2,
                                            _ptr(logits_dev))
    _check(code, ctx.handle)


def uno_spec_step_cohorts(ctx, draft_ids_dev, verify_ids_dev, out_tokens_dev, n_new_dev):
    """One forward: draft rows of draft_ids_dev, verify rows of verify_ids_dev (either may be None)."""
    nd = 0 if draft_ids_dev is None else draft_ids_dev.numel()
    nv = 0 if verify_ids_dev is None else verify_ids_dev.numel()
    code = load_library().uno_spec_step_cohorts(ctx.handle, nd, _ptr(draft_ids_dev) if nd else None, nv,
                                                _ptr(verify_ids_dev) if nv else None,
                                                _ptr(out_tokens_dev) if nv else None,
                                                _ptr(n_new_dev) if nv else None)
    _check(code, ctx.handle)


def uno_spec_step(ctx, req_ids_dev, out_tokens_dev, n_new_dev):
    code = load_library().uno_spec_step(ctx.handle, req_ids_dev.numel(), _ptr(req_ids_dev),
                                        _ptr(out_tokens_dev), _ptr(n_new_dev))
    _check(code, ctx.handle)


def uno_ar_step(ctx, req_ids_dev, out_tokens_dev):
    code = load_library().uno_ar_step(ctx.handle, req_ids_dev.numel(), _ptr(req_ids_dev),
                                      _ptr(out_tokens_dev))
    _check(code, ctx.handle)


def uno_set_graphs(ctx, enable):
    _check(load_library().uno_set_graphs(ctx.handle, int(bool(enable))), ctx.handle)


def uno_set_pdl(ctx, enable):
    _check(load_library().uno_set_pdl(ctx.handle, int(bool(enable))), ctx.handle)


def uno_set_fused(ctx, enable):
    """Returns False when the model does not take the fused pipeline."""
    code = load_library().uno_set_fused(ctx.handle, int(bool(enable)))
    if code == UNO_ERR_UNSUPPORTED:
        return False
    _check(code, ctx.handle)
    return True


def uno_set_verify_split(ctx, max_ctas):
    """spec_verify in its split form above max_ctas (row, chunk) CTAs (0: always)."""
    _check(load_library().uno_set_verify_split(ctx.handle, int(max_ctas)), ctx.handle)


def uno_set_counter_sync(ctx, enable):
    """Fused pipeline: GEMMs wait on completion counters (True) or grid dependencies."""
    _check(load_library().uno_set_counter_sync(ctx.handle, int(bool(enable))), ctx.handle)


def uno_set_tree(ctx, k):
    """Tree sampler with k drafted chains (1: the linear sampler)."""
    _check(load_library().uno_set_tree(ctx.handle, int(k)), ctx.handle)


def uno_set_top_p(ctx, top_p):
    """Nucleus filter of every sampled or verified row (1.0: off)."""
    _check(load_library().uno_set_top_p(ctx.handle, float(top_p)), ctx.handle)


def uno_top_p_filter(logits_dev, top_p, out_dev, stream=None):
    """logits_dev f32 CUDA [rows, vocab] -> out_dev int32 CUDA [rows, 2] (key, id_cut)."""
    rows, vocab = logits_dev.shape
    _check(load_library().uno_top_p_filter(_ptr(logits_dev), rows, vocab, float(top_p),
                                           _ptr(out_dev), _stream_ptr(stream)))


def uno_debug_set_fixed_accept(ctx, a):
    """Benchmark tap: force the accepted length a (first token + accepted
    drafts) of later steps; a <= 0 turns it off."""
    _check(load_library().uno_debug_set_fixed_accept(ctx.handle, int(a)), ctx.handle)


def uno_debug_set_dep_wait(ctx, limit_ns, extra=0):
    """Test tap: counter waits give up after limit_ns; extra > 0 makes them
    unreachable (the step then raises the device flag instead of hanging)."""
    _check(load_library().uno_debug_set_dep_wait(ctx.handle, int(limit_ns), int(extra)), ctx.handle)


def uno_release(ctx, req_id):
    _check(load_library().uno_release(ctx.handle, int(req_id)), ctx.handle)


def uno_destroy(ctx):
    ctx.close()


def uno_last_error(ctx):
    m = load_library().uno_last_error(ctx.handle)
    return m.decode() if m else ""


def uno_status(ctx):
    _check(load_library().uno_status(ctx.handle), ctx.handle)


def uno_request_state(ctx, req_id):
    c, p = ctypes.c_int32(), ctypes.c_int32()
    _check(load_library().uno_request_state(ctx.handle, int(req_id), ctypes.byref(c),
                                            ctypes.byref(p)), ctx.handle)
    return c.value, p.value


def uno_debug_read(ctx, which, out_host):
    """Copy an internal buffer into the host tensor out_host (its size decides the bytes)."""
    nbytes = out_host.numel() * out_host.element_size()
    _check(load_library().uno_debug_read(ctx.handle, which, out_host.data_ptr(), nbytes), ctx.handle)
    return out_host


def uno_debug_kv(ctx, req_id, layer, pos0, n, k_host, v_host):
    _check(load_library().uno_debug_kv(ctx.handle, req_id, layer, pos0, n, k_host.data_ptr(),
                                       v_host.data_ptr()), ctx.handle)


def uno_gated_lora_linear_workspace_bytes(M, N, K, r, dtype):
    return int(load_library().uno_gated_lora_linear_workspace_bytes(M, N, K, r, dtype))


def uno_gated_lora_linear(X, W, A, Bl, gate, scale, Y, workspace, stream=None):
    """Y (f32 CUDA [M, N]) = X W^T + round(gate * scale * X A^T) Bl^T; see include/uno.h."""
    import torch
    dtype = UNO_BF16 if X.dtype == torch.bfloat16 else UNO_F32
    M, K = X.shape
    N = W.shape[0]
    r = A.shape[0] if A is not None else 0
    code = load_library().uno_gated_lora_linear(
        dtype, _ptr(X), _ptr(W), _ptr(A), _ptr(Bl), _ptr(gate), M, N, K, r, scale, _ptr(Y),
        _ptr(workspace), workspace.numel() * workspace.element_size(), _stream_ptr(stream))
    _check(code)


def uno_debug_launch_counts():
    """{'tc_gemm', 'simt_gemm', 'tc_attn', 'simt_attn'}: process-wide launch counts."""
    out = (ctypes.c_int64 * 4)()
    _check(load_library().uno_debug_launch_counts(out))
    return dict(zip(("tc_gemm", "simt_gemm", "tc_attn", "simt_attn"), list(out)))


UNO_K_GEMM, UNO_K_ATTN, UNO_K_SAMPLE, UNO_K_VERIFY, UNO_K_OTHER = range(5)
KERNEL_CLASSES = ("gemm", "attn", "sample", "verify", "other")


def uno_profile_begin(ctx, class_mask):
    _check(load_library().uno_profile_begin(ctx.handle, int(class_mask)), ctx.handle)


def uno_profile_end(ctx):
    """Returns {class: (launches, ms, algorithmic bytes)}."""
    n = len(KERNEL_CLASSES)
    launches, ms, nbytes = (ctypes.c_int64 * n)(), (ctypes.c_double * n)(), (ctypes.c_double * n)()
    _check(load_library().uno_profile_end(ctx.handle, launches, ms, nbytes), ctx.handle)
    return {k: (launches[i], ms[i], nbytes[i]) for i, k in enumerate(KERNEL_CLASSES)}


class UnoProfRecord(ctypes.Structure):
    _fields_ = [("cls", ctypes.c_int32), ("m", ctypes.c_int32), ("n", ctypes.c_int32),
                ("k", ctypes.c_int32), ("r", ctypes.c_int32), ("ms", ctypes.c_float)]


def uno_profile_records(ctx):
    """Per-launch records of the last uno_profile_end: list of dicts."""
    lib = load_library()
    n = lib.uno_profile_records(ctx.handle, None, 0)
    if n < 0:
        _check(-n, ctx.handle)
    arr = (UnoProfRecord * max(n, 1))()
    lib.uno_profile_records(ctx.handle, arr, n)
    return [{"cls": KERNEL_CLASSES[a.cls], "m": a.m, "n": a.n, "k": a.k, "r": a.r, "ms": a.ms}
            for a in arr[:n]]


def uno_spec_verify_workspace_bytes(n_req, n_tests, vocab):
    return int(load_library().uno_spec_verify_workspace_bytes(n_req, n_tests, vocab))


def uno_spec_verify(p_dev, q_dev, drafts_dev, seed, streams_dev, pos0_dev, out_tokens_dev,
                    n_out_dev, workspace_dev, stream=None):
    """p_dev, q_dev: f32 CUDA [n_req, n_tests, vocab]; see include/uno.h."""
    n_req, n_tests, vocab = p_dev.shape
    code = load_library().uno_spec_verify(
        _ptr(p_dev), _ptr(q_dev), _ptr(drafts_dev), n_req, n_tests, vocab, seed, _ptr(streams_dev),
        _ptr(pos0_dev), _ptr(out_tokens_dev), _ptr(n_out_dev), _ptr(workspace_dev),
        workspace_dev.numel() * workspace_dev.element_size(), _stream_ptr(stream))
    _check(code)


def uno_spec_verify_noalloc_max_bytes():
    return int(load_library().uno_spec_verify_noalloc_max_bytes())


def uno_spec_verify_noalloc(p_dev, q_dev, drafts_dev, seed, streams_dev, pos0_dev, out_tokens_dev,
                            n_out_dev, stream=None):
    """uno_spec_verify with the library's fixed scratch array instead of a
    workspace (for callers that cannot allocate device memory)."""
    n_req, n_tests, vocab = p_dev.shape
    code = load_library().uno_spec_verify_noalloc(
        _ptr(p_dev), _ptr(q_dev), _ptr(drafts_dev), n_req, n_tests, vocab, seed, _ptr(streams_dev),
        _ptr(pos0_dev), _ptr(out_tokens_dev), _ptr(n_out_dev), _stream_ptr(stream))
    _check(code)
