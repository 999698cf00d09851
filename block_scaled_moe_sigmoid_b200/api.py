"""Thin ctypes binding to ``libmoe_sm100.so`` (include/moe.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch supplies device memory and the current CUDA stream.  There is
no fallback: if the library is missing or cannot load, every call raises.
"""
import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe_sm100.so")

MOE_OK = 0
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED_SHAPE",
                3: "MOE_ERR_ALIGNMENT", 4: "MOE_ERR_CUDA", 5: "MOE_ERR_TIMEOUT",
                6: "MOE_ERR_NOT_INITIALIZED", 7: "MOE_ERR_DEVICE_FAULT"}

# exported symbols and their argument types (ctypes)
_P, _I, _S = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
# moe_bias_rule_t: (quantiles, n_levels, E, bias, bias_next, stream, user)
BIAS_RULE = ctypes.CFUNCTYPE(None, _P, _I, _I, _P, _P, _P, _P)
SIGNATURES = {
    "moe_plan_create": [_I, _I, _I, _I, _I, _I, _I, _I, _I, ctypes.POINTER(_P)],
    "moe_plan_workspace_bytes": [_P, ctypes.POINTER(_S)],
    "moe_plan_set_workspace": [_P, _P, _S],
    "moe_plan_check": [_P, _P, ctypes.POINTER(ctypes.c_uint)],
    "moe_plan_destroy": [_P],
    "moe_status_string": [_I],
    "moe_quant_mxfp8": [_P, _I, _I, _P, _P, _P],
    "moe_route": [_P, _P, _I, _P, _P, _P, _P, _P, _P],
    "moe_permute": [_P, _P, _I, _P, _P, _P, _P, _P],
    "moe_forward": [_P, _P, _I, _P, _P, _P, _P, _P, _P],
    "moe_expert_bytes": [_I, _I, _I, ctypes.POINTER(_S), ctypes.POINTER(_S), ctypes.POINTER(_S),
                         ctypes.POINTER(_S)],
    "moe_pack_expert_mxfp4": [_I, _I, _I, _P, _P, _P, _P, _P],
    "moe_pack_shared_bf16": [_I, _I, _P, _P, _P, _P, _P],
    "moe_debug_buffer": [_P, _I, ctypes.POINTER(_P), ctypes.POINTER(_S)],
    "moe_debug_timeout_probe": [_P, _P],
    "moe_plan_set_latent": [_P, _I, ctypes.c_float],
    "moe_forward_latent": [_P, _P, _I, _P, _P, _P, _P, _P, _P, _P],
    "moe_plan_set_profiling": [_P, _I],
    "moe_plan_set_option": [_P, _I, _I],
    "moe_plan_get_option": [_P, _I, ctypes.POINTER(_I)],
    "moe_permute_noalloc": [_P, _I, _I, _I, _P, _P, _P, _P, _P],
    "moe_plan_stage_ms": [_P, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_int), _I],
    "moe_route_margin_quantiles": [_P, _P, _P, _I, ctypes.POINTER(ctypes.c_double), _I, _P, _P],
    "moe_quantile_balance": [_P, _P, _P, _I, ctypes.POINTER(ctypes.c_double), _I, BIAS_RULE, _P, _P, _P],
}


STAGES = ["router_split", "router_gemm", "topk", "permute", "quant_scatter", "gate_up_glu",
          "down", "shared_gate_up", "shared_down", "combine", "latent_in", "latent_out"]
# kernel launches per recorded stage instance ("topk" is the selection kernel, which also
# sums the router GEMM's K-split partials)
STAGE_KERNELS = {"permute": 3, "quant_scatter": 2, "latent_in": 2, "latent_out": 2}


class MoeError(RuntimeError):
    def __init__(self, fn, code):
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(code, code)}")
        self.code = code


class ExpertsMXFP4(ctypes.Structure):
    _fields_ = [("w_gu", _P), ("s_gu", _P), ("w_dn", _P), ("s_dn", _P)]


class SharedBF16(ctypes.Structure):
    _fields_ = [("w_gu", _P), ("w_dn", _P)]


class LatentBF16(ctypes.Structure):
    _fields_ = [("w_down", _P), ("gamma", _P), ("w_up", _P)]


_lib = None


def lib():
    """Load the library (raises if it is missing: there is no CPU fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m block_scaled_moe_sigmoid_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, argtypes in SIGNATURES.items():
            fn = getattr(L, name)
            fn.argtypes = argtypes
            fn.restype = ctypes.c_char_p if name == "moe_status_string" else ctypes.c_int
        _lib = L
    return _lib


def _call(name, *args):
    code = getattr(lib(), name)(*args)
    if code != MOE_OK:
        raise MoeError(name, code)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


# ------------------------------------------------------------------ same names as the C ABI
def moe_plan_create(T_max, d, E, k, I, I_shared=0, act=0, bias_mode=0, flags=0):
    h = ctypes.c_void_p()
    _call("moe_plan_create", T_max, d, E, k, I, I_shared, act, bias_mode, flags, ctypes.byref(h))
    return h


def moe_plan_workspace_bytes(plan):
    n = ctypes.c_size_t()
    _call("moe_plan_workspace_bytes", plan, ctypes.byref(n))
    return n.value


def moe_plan_set_workspace(plan, ws):
    _call("moe_plan_set_workspace", plan, _ptr(ws), ws.numel() * ws.element_size())


def moe_plan_check(plan, stream=None):
    bits = ctypes.c_uint()
    code = lib().moe_plan_check(plan, _stream(stream), ctypes.byref(bits))
    return code, bits.value


def moe_debug_timeout_probe(plan, stream=None):
    """One bounded wait that runs out on the GPU (see include/moe.h)."""
    _call("moe_debug_timeout_probe", plan, _stream(stream))


def moe_plan_destroy(plan):
    _call("moe_plan_destroy", plan)


def moe_quant_mxfp8(x, q=None, scale=None, stream=None):
    """x: cuda bf16 [rows, cols] -> (q uint8 [rows, cols], scale uint8 [rows, cols/32])."""
    rows, cols = x.shape
    q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device) if q is None else q
    scale = torch.empty((rows, cols // 32), dtype=torch.uint8, device=x.device) if scale is None else scale
    _call("moe_quant_mxfp8", _ptr(x), rows, cols, _ptr(q), _ptr(scale), _stream(stream))
    return q, scale


def moe_route(plan, x, W_r, bias, k, idx=None, w=None, logits=None, stream=None):
    T = x.shape[0]
    idx = torch.empty((T, k), dtype=torch.int32, device=x.device) if idx is None else idx
    w = torch.empty((T, k), dtype=torch.float32, device=x.device) if w is None else w
    _call("moe_route", plan, _ptr(x), T, _ptr(W_r), _ptr(bias), _ptr(idx), _ptr(w), _ptr(logits),
          _stream(stream))
    return idx, w


def moe_permute(plan, idx, E, stream=None):
    T, k = idx.shape
    dev = idx.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm_tok = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty((T, k), dtype=torch.int32, device=dev)
    _call("moe_permute", plan, _ptr(idx), T, _ptr(counts), _ptr(offsets), _ptr(perm_tok), _ptr(inv),
          _stream(stream))
    return counts, offsets, perm_tok, inv


def moe_permute_noalloc(idx, E, stream=None):
    """moe_permute for callers that cannot allocate device memory: the library uses its own
    fixed device scratch array (see include/moe.h for the size limit).  The output
    tensors here are allocated by torch for convenience."""
    T, k = idx.shape
    dev = idx.device
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    perm_tok = torch.empty(T * k, dtype=torch.int32, device=dev)
    inv = torch.empty((T, k), dtype=torch.int32, device=dev)
    _call("moe_permute_noalloc", _ptr(idx), T, E, k, _ptr(counts), _ptr(offsets), _ptr(perm_tok),
          _ptr(inv), _stream(stream))
    return counts, offsets, perm_tok, inv


def moe_forward(plan, x, idx, w, experts, shared, y=None, stream=None):
    T, d = x.shape
    y = torch.empty((T, d), dtype=torch.bfloat16, device=x.device) if y is None else y
    ex = experts.struct()
    sh = shared.struct() if shared is not None else None
    _call("moe_forward", plan, _ptr(x), T, _ptr(idx), _ptr(w), ctypes.byref(ex),
          ctypes.byref(sh) if sh is not None else None, _ptr(y), _stream(stream))
    return y


def moe_forward_latent(plan, x, idx, w, latent, experts, shared, y=None, stream=None):
    T, d = x.shape
    y = torch.empty((T, d), dtype=torch.bfloat16, device=x.device) if y is None else y
    lat = latent.struct()
    ex = experts.struct()
    sh = shared.struct() if shared is not None else None
    _call("moe_forward_latent", plan, _ptr(x), T, _ptr(idx), _ptr(w), ctypes.byref(lat), ctypes.byref(ex),
          ctypes.byref(sh) if sh is not None else None, _ptr(y), _stream(stream))
    return y


def moe_route_margin_quantiles(plan, logits, E, levels, select_bias=None, quantiles=None, stream=None):
    """Per-expert quantiles of the routing margins of logits [T, E] (fp32, device) at the
    given levels; returns fp32 [len(levels), E] on the device."""
    T = logits.shape[0]
    lv = (ctypes.c_double * len(levels))(*levels)
    if quantiles is None:
        quantiles = torch.empty((len(levels), E), dtype=torch.float32, device=logits.device)
    _call("moe_route_margin_quantiles", plan, _ptr(logits), _ptr(select_bias), T, lv, len(levels),
          _ptr(quantiles), _stream(stream))
    return quantiles


def moe_quantile_balance(plan, logits, bias, levels, rule, bias_next=None, user=None, stream=None):
    """Margin quantiles of this step, then the caller's rule (a BIAS_RULE callable) writes the
    next step's bias into bias_next (fp32 [E], device)."""
    T = logits.shape[0]
    lv = (ctypes.c_double * len(levels))(*levels)
    if bias_next is None:
        bias_next = torch.empty_like(bias)
    _call("moe_quantile_balance", plan, _ptr(logits), _ptr(bias), T, lv, len(levels), rule, user,
          _ptr(bias_next), _stream(stream))
    return bias_next


def moe_expert_bytes(d, I, E):
    a, b, c, e = (ctypes.c_size_t() for _ in range(4))
    _call("moe_expert_bytes", d, I, E, ctypes.byref(a), ctypes.byref(b), ctypes.byref(c), ctypes.byref(e))
    return a.value, b.value, c.value, e.value


def moe_pack_expert_mxfp4(d, I, e, w_gate, w_up, w_down, experts, stream=None):
    ex = experts.struct()
    _call("moe_pack_expert_mxfp4", d, I, e, _ptr(w_gate), _ptr(w_up), _ptr(w_down), ctypes.byref(ex),
          _stream(stream))


def moe_pack_shared_bf16(d, I_shared, w_gate, w_up, w_down, shared, stream=None):
    sh = shared.struct()
    _call("moe_pack_shared_bf16", d, I_shared, _ptr(w_gate), _ptr(w_up), _ptr(w_down), ctypes.byref(sh),
          _stream(stream))


def moe_debug_buffer(plan, which):
    """(device pointer, bytes) of a workspace buffer (see include/moe.h)."""
    p, n = ctypes.c_void_p(), ctypes.c_size_t()
    _call("moe_debug_buffer", plan, which, ctypes.byref(p), ctypes.byref(n))
    return p.value, n.value


MOE_OPT_PREFETCH_DIST, MOE_OPT_PREFETCH_B, MOE_OPT_TILE_N, MOE_OPT_ROUTER_SPLIT = 0, 1, 2, 3
MOE_OPT_SHARED_SPLIT, MOE_OPT_SHARED_SPLIT_DOWN = 4, 5


def moe_plan_set_option(plan, option, value):
    _call("moe_plan_set_option", plan, option, int(value))


def moe_plan_get_option(plan, option):
    v = ctypes.c_int()
    _call("moe_plan_get_option", plan, option, ctypes.byref(v))
    return v.value


def moe_plan_set_profiling(plan, enable=True):
    _call("moe_plan_set_profiling", plan, 1 if enable else 0)


def moe_plan_stage_ms(plan):
    """{stage: (summed ms, recorded launches)} since profiling was enabled / last queried."""
    n = len(STAGES)
    ms = (ctypes.c_float * n)()
    cnt = (ctypes.c_int * n)()
    _call("moe_plan_stage_ms", plan, ms, cnt, n)
    return {STAGES[i]: (ms[i], cnt[i]) for i in range(n)}


# ------------------------------------------------------------------ buffers
class Experts:
    """Device buffers of packed MXFP4 experts (allocated by torch)."""

    def __init__(self, d, I, E, device="cuda"):
        self.d, self.I, self.E = d, I, E
        sizes = moe_expert_bytes(d, I, E)
        # 256-byte aligned allocations (torch's caching allocator returns 512-aligned blocks)
        self.w_gu, self.s_gu, self.w_dn, self.s_dn = (
            torch.empty(n, dtype=torch.uint8, device=device) for n in sizes)

    def struct(self):
        return ExpertsMXFP4(self.w_gu.data_ptr(), self.s_gu.data_ptr(), self.w_dn.data_ptr(),
                            self.s_dn.data_ptr())

    def pack(self, e, w_gate, w_up, w_down, stream=None):
        moe_pack_expert_mxfp4(self.d, self.I, e, w_gate.contiguous(), w_up.contiguous(),
                              w_down.contiguous(), self, stream)


class Shared:
    def __init__(self, d, I_shared, device="cuda"):
        self.d, self.I_shared = d, I_shared
        self.w_gu = torch.empty((2 * I_shared, d), dtype=torch.bfloat16, device=device)
        self.w_dn = torch.empty((d, I_shared), dtype=torch.bfloat16, device=device)

    def struct(self):
        return SharedBF16(self.w_gu.data_ptr(), self.w_dn.data_ptr())

    def pack(self, w_gate, w_up, w_down, stream=None):
        moe_pack_shared_bf16(self.d, self.I_shared, w_gate.contiguous(), w_up.contiguous(),
                             w_down.contiguous(), self, stream)


MOE_ACT_SILU_GLU, MOE_ACT_CLAMPED_SWIGLU = 0, 1
MOE_BIAS_LOGIT, MOE_BIAS_SELECT_ONLY = 0, 1
MOE_FLAG_STATIC_ROUTER = 1


class Latent:
    """Latent-option weights on the device: W_ld bf16 [d_latent][d], gamma fp32 [d_latent],
    W_lu bf16 [d][d_latent]."""

    def __init__(self, w_down, gamma, w_up):
        self.w_down = w_down.to(torch.bfloat16).contiguous()
        self.gamma = gamma.to(torch.float32).contiguous()
        self.w_up = w_up.to(torch.bfloat16).contiguous()

    def struct(self):
        return LatentBF16(self.w_down.data_ptr(), self.gamma.data_ptr(), self.w_up.data_ptr())


class Plan:
    """A plan plus its torch-allocated workspace."""

    def __init__(self, T_max, d, E, k, I, I_shared=0, device="cuda", act=MOE_ACT_SILU_GLU,
                 bias_mode=MOE_BIAS_LOGIT, flags=0, d_latent=0, eps=1e-5):
        self.T_max, self.d, self.E, self.k, self.I, self.I_shared = T_max, d, E, k, I, I_shared
        self.act, self.bias_mode, self.flags, self.d_latent = act, bias_mode, flags, d_latent
        self.handle = moe_plan_create(T_max, d, E, k, I, I_shared, act, bias_mode, flags)
        if d_latent:
            _call("moe_plan_set_latent", self.handle, d_latent, ctypes.c_float(eps))
        n = moe_plan_workspace_bytes(self.handle)
        self.workspace = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
        moe_plan_set_workspace(self.handle, self.workspace)

    def route(self, x, W_r, bias=None, logits=None, stream=None):
        return moe_route(self.handle, x, W_r, bias, self.k, logits=logits, stream=stream)

    def permute(self, idx, stream=None):
        return moe_permute(self.handle, idx, self.E, stream)

    def forward(self, x, idx, w, experts, shared=None, y=None, stream=None, latent=None):
        if self.d_latent:
            return moe_forward_latent(self.handle, x, idx, w, latent, experts, shared, y, stream)
        return moe_forward(self.handle, x, idx, w, experts, shared, y, stream)

    def check(self, stream=None):
        return moe_plan_check(self.handle, stream)

    def debug_tensor(self, which, dtype, shape):
        """A torch view of a workspace buffer (copy it before the next call)."""
        ptr, n = moe_debug_buffer(self.handle, which)
        off = ptr - self.workspace.data_ptr()
        count = 1
        for s in shape:
            count *= s
        nbytes = count * torch.empty((), dtype=dtype).element_size()
        assert 0 <= off and nbytes <= n
        return self.workspace[off:off + nbytes].view(dtype).view(*shape)

    def __del__(self):
        try:
            if getattr(self, "handle", None) is not None:
                moe_plan_destroy(self.handle)
                self.handle = None
        except Exception:
            pass
