"""ctypes binding of libmoe.so (the C ABI in include/moe.h).

Argument marshalling only: every step of the layer runs in the library's
CUDA kernels. PyTorch supplies device memory and the current stream.
Importing this module loads the library and raises ImportError if it has
not been built (``python -m mixture_experts_layer_33_b200.build``); calls
raise RuntimeError with the library's status string when a call fails.
With MOE_DEBUG=1 in the environment it loads the MOE_DEBUG build
(``libmoe_debug.so``, ``build --debug``) instead: the same entry points,
whose kernels also range-check the indices callers hand in.
"""

from __future__ import annotations

import ctypes
import os

import torch

DEBUG_BUILD = os.environ.get("MOE_DEBUG", "0") == "1"
_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)),
                         "libmoe_debug.so" if DEBUG_BUILD else "libmoe.so")

MOE_OK = 0
F32, BF16 = 0, 1
TOKEN_TOPK, EXPERT_CHOICE, DES_VOTE, DES_SEQ = 0, 1, 2, 3
GELU_ERF, SWIGLU = 0, 1
HEAVY, IDENTITY, ZERO, CONST = 0, 1, 2, 3
DEV_BAD_EXPERT, DEV_BAD_TOKEN, DEV_TIMEOUT, DEV_OVERFLOW, DEV_BAD_INDEX = 1, 2, 4, 8, 16
BUILD_DEBUG = 1  # moe_build_flags() bit of the MOE_DEBUG build
MAX_EXPERTS = 256

# Names of every entry point include/moe.h declares.
ENTRY_POINTS = (
    "moe_status_string", "moe_device_check", "moe_num_assignments",
    "moe_workspace_size", "moe_router", "moe_select_topk",
    "moe_select_expert_choice", "moe_core_set_vote", "moe_core_set_union", "moe_dispatch",
    "moe_grouped_mlp", "moe_combine", "moe_forward", "moe_forward_host",
    "moe_dispatch_noalloc", "moe_activation", "moe_test_set_barrier_wait", "moe_build_flags",
)
NOALLOC_SCRATCH_BYTES = 256 * 1024  # MOE_NOALLOC_SCRATCH_BYTES


class MoeConfig(ctypes.Structure):
    _fields_ = [
        ("T", ctypes.c_int32), ("d", ctypes.c_int32), ("h", ctypes.c_int32),
        ("E", ctypes.c_int32), ("n_heavy", ctypes.c_int32), ("k", ctypes.c_int32),
        ("n_shared", ctypes.c_int32), ("h_shared", ctypes.c_int32),
        ("dtype", ctypes.c_int32), ("act", ctypes.c_int32), ("routing", ctypes.c_int32),
        ("group_size", ctypes.c_int32), ("capacity", ctypes.c_int32), ("M_core", ctypes.c_int32),
        ("gate_residual_scale", ctypes.c_float), ("renorm", ctypes.c_int32),
        ("k_local", ctypes.c_int32), ("const_mix", ctypes.c_int32),
        ("expert_kind", ctypes.c_int32 * MAX_EXPERTS),
    ]


class MoeForwardAux(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in
                ("logits", "probs", "sel", "w", "votes", "core", "offsets")]


_vp, _i32, _f32, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
_CFG = ctypes.POINTER(MoeConfig)
_SIGS = {
    "moe_status_string": (ctypes.c_char_p, [_i32]),
    "moe_device_check": (_i32, [_i32]),
    "moe_num_assignments": (_i32, [_CFG, ctypes.POINTER(ctypes.c_int64)]),
    "moe_workspace_size": (_i32, [_CFG, ctypes.POINTER(_sz)]),
    "moe_router": (_i32, [_vp, _vp, _vp, _vp, _f32, _i32, _i32, _i32, _i32, _vp, _vp, _i32, _i32,
                          _vp, _vp, _vp]),
    "moe_select_topk": (_i32, [_vp, _vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_select_expert_choice": (_i32, [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp]),
    "moe_core_set_vote": (_i32, [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "moe_core_set_union": (_i32, [_vp, _i32, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp]),
    "moe_dispatch": (_i32, [_CFG, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp]),
    "moe_dispatch_noalloc": (_i32, [_CFG, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "moe_activation": (_i32, [_vp, _vp, ctypes.c_int64, _i32, _vp]),
    "moe_test_set_barrier_wait": (_i32, [ctypes.c_uint64, _i32]),
    "moe_build_flags": (_i32, []),
    "moe_grouped_mlp": (_i32, [_CFG, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz,
                               _vp]),
    "moe_combine": (_i32, [_CFG, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                           _vp]),
    "moe_forward": (_i32, [_CFG, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                           ctypes.POINTER(MoeForwardAux), _vp, _vp, _sz, _vp]),
    "moe_forward_host": (_i32, [_CFG, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp,
                                _vp, _sz, _vp]),
}


def _load():
    if not os.path.exists(_LIB_PATH):
        raise ImportError(
            f"{_LIB_PATH} is not built; run `python -m mixture_experts_layer_33_b200.build`")
    lib = ctypes.CDLL(_LIB_PATH)
    for name, (res, args) in _SIGS.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = _load()
LIB_PATH = _LIB_PATH


def build_flags():
    """MOE_BUILD_* bits of the loaded library (BUILD_DEBUG: the MOE_DEBUG build)."""
    return LIB.moe_build_flags()


def status_string(code):
    return LIB.moe_status_string(int(code)).decode()


def _check(code, what):
    if code != MOE_OK:
        raise RuntimeError(f"{what} failed: {status_string(code)}")


def _ptr(t):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return t.data_ptr()


def _dev_ptr(t):
    if t is not None and not t.is_cuda:
        raise ValueError("device tensor expected")
    return _ptr(t)


def _stream(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


# ------------------------------------------------------------------ config
def make_config(cfg) -> MoeConfig:
    """MoeConfig from a workload dict (see ``inputs.WORKLOADS``)."""
    c = MoeConfig()
    kinds = list(cfg.get("kinds", [HEAVY] * cfg["E"]))
    c.T, c.d, c.h, c.E = cfg["T"], cfg["d"], cfg["h"], cfg["E"]
    c.n_heavy = sum(1 for k in kinds if k == HEAVY)
    c.k = cfg.get("k", 0)
    c.n_shared, c.h_shared = cfg.get("n_shared", 0), cfg.get("h_shared", 0)
    c.dtype = BF16 if cfg["dtype"] == "bf16" else F32
    c.act = SWIGLU if cfg["act"] == "swiglu" else GELU_ERF
    c.routing = {"token_topk": TOKEN_TOPK, "expert_choice": EXPERT_CHOICE,
                 "des_vote": DES_VOTE, "des_seq": DES_SEQ}[cfg["routing"]]
    c.group_size = cfg.get("group_size", 0)
    c.capacity = cfg.get("capacity", 0)
    c.M_core = cfg.get("M_core", 0)
    c.gate_residual_scale = float(cfg.get("gate_residual_scale", 0.0))
    c.renorm = int(cfg.get("renorm", 0))
    c.k_local = int(cfg.get("k_local", 0))
    c.const_mix = int(cfg.get("const_mix", 0))
    for e, k in enumerate(kinds):
        c.expert_kind[e] = k
    return c


def num_assignments(c: MoeConfig) -> int:
    n = ctypes.c_int64()
    _check(LIB.moe_num_assignments(ctypes.byref(c), ctypes.byref(n)), "moe_num_assignments")
    return n.value


def workspace_size(c: MoeConfig) -> int:
    n = _sz()
    _check(LIB.moe_workspace_size(ctypes.byref(c), ctypes.byref(n)), "moe_workspace_size")
    return n.value


def alloc_workspace(c: MoeConfig, device="cuda"):
    """A caller-owned workspace of moe_workspace_size() bytes (256-byte aligned)."""
    return torch.empty(workspace_size(c), dtype=torch.uint8, device=device)


def device_check(device=0):
    return LIB.moe_device_check(int(device))


# ------------------------------------------------------------- entry points
def router(x, W_r, logits, probs, bias=None, z_prev=None, z_prev_scale=0.0, k=0, renorm=0,
           idx=None, w=None, stream=None):
    T, d = x.shape
    E = W_r.shape[0]
    dt = BF16 if x.dtype == torch.bfloat16 else F32
    _check(LIB.moe_router(_dev_ptr(x), _dev_ptr(W_r), _dev_ptr(bias), _dev_ptr(z_prev),
                          float(z_prev_scale), T, d, E, dt, _dev_ptr(logits), _dev_ptr(probs),
                          int(k), int(renorm), _dev_ptr(idx), _dev_ptr(w), _stream(stream)),
           "moe_router")


def select_topk(logits, probs, k, idx, w, renorm=0, stream=None):
    T, E = logits.shape
    _check(LIB.moe_select_topk(_dev_ptr(logits), _dev_ptr(probs), T, E, int(k), int(renorm),
                               _dev_ptr(idx), _dev_ptr(w), _stream(stream)), "moe_select_topk")


def select_expert_choice(probs, group_size, C, tok, w, stream=None):
    T, E = probs.shape
    _check(LIB.moe_select_expert_choice(_dev_ptr(probs), T, E, int(group_size), int(C),
                                        _dev_ptr(tok), _dev_ptr(w), _stream(stream)),
           "moe_select_expert_choice")


def core_set_vote(probs, K, M_core, votes, core, idx, w, stream=None):
    N, M = probs.shape
    _check(LIB.moe_core_set_vote(_dev_ptr(probs), N, M, int(K), int(M_core), _dev_ptr(votes),
                                 _dev_ptr(core), _dev_ptr(idx), _dev_ptr(w), _stream(stream)),
           "moe_core_set_vote")


def core_set_union(probs, K, k_local, core, n_core, idx, w, stream=None):
    N, M = probs.shape
    _check(LIB.moe_core_set_union(_dev_ptr(probs), N, M, int(K), int(k_local), _dev_ptr(core),
                                  _dev_ptr(n_core), _dev_ptr(idx), _dev_ptr(w), _stream(stream)),
           "moe_core_set_union")


def dispatch(c: MoeConfig, sel, x, x_perm, offsets, perm, row_of, tok_ptr, tok_assign,
             dev_status, ws, stream=None):
    _check(LIB.moe_dispatch(ctypes.byref(c), _dev_ptr(sel), _dev_ptr(x), _dev_ptr(x_perm),
                            _dev_ptr(offsets), _dev_ptr(perm), _dev_ptr(row_of),
                            _dev_ptr(tok_ptr), _dev_ptr(tok_assign), _dev_ptr(dev_status),
                            _dev_ptr(ws), ws.numel(), _stream(stream)), "moe_dispatch")


def dispatch_noalloc(c: MoeConfig, sel, x, x_perm, offsets, perm, row_of, tok_ptr, tok_assign,
                     dev_status, stream=None):
    """moe_dispatch for callers that cannot allocate device memory.

    Same arguments and outputs as ``dispatch`` minus the workspace: the
    library keeps the histogram scratch in a fixed device array of
    NOALLOC_SCRATCH_BYTES per GPU. Configurations whose scratch would not
    fit (ceil(n_assign/1024) * n_heavy * 4 bytes) are rejected. The first
    call on a device sets up the array's address (make it before any stream
    capture); calls that overlap on the GPU share the array and race.
    """
    code = LIB.moe_dispatch_noalloc(ctypes.byref(c), _dev_ptr(sel), _dev_ptr(x),
                                    _dev_ptr(x_perm), _dev_ptr(offsets), _dev_ptr(perm),
                                    _dev_ptr(row_of), _dev_ptr(tok_ptr), _dev_ptr(tok_assign),
                                    _dev_ptr(dev_status), _stream(stream))
    if code == 2:
        raise RuntimeError(
            "moe_dispatch_noalloc failed: the configuration's dispatch scratch "
            f"(ceil(n_assign/1024) * n_heavy * 4 bytes) exceeds the {NOALLOC_SCRATCH_BYTES}-byte "
            "library-owned array; use dispatch() with a workspace")
    _check(code, "moe_dispatch_noalloc")


def activation(x, y, act=GELU_ERF, stream=None):
    """y = GELU(x) (act=GELU_ERF) or SiLU(x) (act=SWIGLU), fp32 device tensors."""
    _check(LIB.moe_activation(_dev_ptr(x), _dev_ptr(y), x.numel(), int(act), _stream(stream)),
           "moe_activation")


def set_barrier_wait_for_tests(limit_ns=0, extra_arrivals=0):
    """Test hook: the small-block routing kernel's grid-barrier wait limit
    (ns; 0 = the 2 s default) and extra arrivals it waits for (0 = none).
    Process-wide; see moe_test_set_barrier_wait in include/moe.h."""
    _check(LIB.moe_test_set_barrier_wait(int(limit_ns), int(extra_arrivals)),
           "moe_test_set_barrier_wait")


def grouped_mlp(c: MoeConfig, x_perm, offsets, W1, W2, x, Ws1, Ws2, y_perm, y_shared,
                dev_status, ws, stream=None):
    _check(LIB.moe_grouped_mlp(ctypes.byref(c), _dev_ptr(x_perm), _dev_ptr(offsets),
                               _dev_ptr(W1), _dev_ptr(W2), _dev_ptr(x), _dev_ptr(Ws1),
                               _dev_ptr(Ws2), _dev_ptr(y_perm), _dev_ptr(y_shared),
                               _dev_ptr(dev_status), _dev_ptr(ws), ws.numel(), _stream(stream)),
           "moe_grouped_mlp")


def combine(c: MoeConfig, y_perm, y_shared, sel, w, row_of, tok_ptr, tok_assign, x, const_vecs,
            residual, y, dev_status, stream=None):
    _check(LIB.moe_combine(ctypes.byref(c), _dev_ptr(y_perm), _dev_ptr(y_shared), _dev_ptr(sel),
                           _dev_ptr(w), _dev_ptr(row_of), _dev_ptr(tok_ptr),
                           _dev_ptr(tok_assign), _dev_ptr(x), _dev_ptr(const_vecs),
                           _dev_ptr(residual), _dev_ptr(y), _dev_ptr(dev_status),
                           _stream(stream)), "moe_combine")


def forward(c: MoeConfig, x, W_r, W1, W2, y, ws, residual=None, z_prev=None, bias=None,
            Ws1=None, Ws2=None, const_vecs=None, aux=None, dev_status=None, stream=None):
    """The whole layer on device buffers. ``aux`` is a dict of optional
    output tensors (logits, probs, sel, w, votes, core, offsets)."""
    a = None
    if aux:
        a = MoeForwardAux(*[_dev_ptr(aux.get(n)) for n, _ in MoeForwardAux._fields_])
    _check(LIB.moe_forward(ctypes.byref(c), _dev_ptr(x), _dev_ptr(residual), _dev_ptr(z_prev),
                           _dev_ptr(W_r), _dev_ptr(bias), _dev_ptr(W1), _dev_ptr(W2),
                           _dev_ptr(Ws1), _dev_ptr(Ws2), _dev_ptr(const_vecs), _dev_ptr(y),
                           ctypes.byref(a) if a is not None else None, _dev_ptr(dev_status),
                           _dev_ptr(ws), ws.numel(), _stream(stream)), "moe_forward")


def forward_host(c: MoeConfig, x_host, W_r, W1, W2, y_host, ws, residual_host=None,
                 z_prev_host=None, bias=None, Ws1=None, Ws2=None, const_vecs=None,
                 dev_status=None, stream=None):
    """The whole layer with x / residual / z_prev / y in host memory (pin
    them for asynchronous copies); weights stay on the device."""
    for t in (x_host, y_host, residual_host, z_prev_host):
        if t is not None and t.is_cuda:
            raise ValueError("host tensor expected")
    _check(LIB.moe_forward_host(ctypes.byref(c), _ptr(x_host), _ptr(residual_host),
                                _ptr(z_prev_host), _dev_ptr(W_r), _dev_ptr(bias), _dev_ptr(W1),
                                _dev_ptr(W2), _dev_ptr(Ws1), _dev_ptr(Ws2),
                                _dev_ptr(const_vecs), _ptr(y_host), _dev_ptr(dev_status),
                                _dev_ptr(ws), ws.numel(), _stream(stream)), "moe_forward_host")


class MoELayer:
    """A configured layer: weights and a workspace resident on one device.

    ``layer(x, z_prev=None)`` returns y; ``residual`` defaults to x.
    """

    def __init__(self, cfg, weights, device="cuda"):
        self.cfg = cfg
        self.c = make_config(cfg)
        self.w = weights
        self.ws = alloc_workspace(self.c, device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)

    def __call__(self, x, z_prev=None, residual="x", aux=None, stream=None):
        y = torch.empty_like(x)
        res = x if residual == "x" else residual
        w = self.w
        forward(self.c, x, w["W_r"], w["W1"], w["W2"], y, self.ws, residual=res, z_prev=z_prev,
                bias=w.get("logit_bias"), Ws1=w.get("Ws1"), Ws2=w.get("Ws2"),
                const_vecs=w.get("const_vecs"), aux=aux, dev_status=self.status, stream=stream)
        return y
