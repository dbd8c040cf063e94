"""Python binding of libvsa.so (argument marshalling only).

Every step of the forward pass runs in the library's CUDA kernels; PyTorch
only provides device memory and the current stream. There is no CPU path:
calls raise if the library is not built or the tensors are not on an
sm_100 CUDA device.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
lib_path = os.path.join(HERE, "libvsa.so")

STATUS = {0: "VSA_OK", 1: "VSA_ERR_INVALID_ARG", 2: "VSA_ERR_SHAPE", 3: "VSA_ERR_UNSUPPORTED",
          4: "VSA_ERR_ALIGN", 5: "VSA_ERR_CUDA", 6: "VSA_ERR_TIMEOUT", 7: "VSA_ERR_DEVICE"}

EXPORTED = ["vsa_workspace_bytes", "vsa_workspace_layout", "vsa_plan", "vsa_run", "vsa_run_fixed_idx",
            "vsa_forward", "vsa_check", "vsa_plan_destroy", "vsa_status_string", "vsa_set_wait_limit_ns",
            "vsa_set_debug_stall", "vsa_set_stage_timing", "vsa_stage_times", "vsa_kernels_per_run",
            "vsa_forward_noalloc", "vsa_set_cube_major_copies", "vsa_run_host", "vsa_measure_l2_read",
            "vsa_run_train", "vsa_backward_workspace_bytes", "vsa_run_backward", "vsa_backward_stage_times",
            "vsa_stage_times_history", "vsa_backward_stage_times_history"]


class VSAError(RuntimeError):
    def __init__(self, code: int, what: str = ""):
        self.code = code
        super().__init__(f"{what}: {STATUS.get(code, code)}" if what else STATUS.get(code, str(code)))


class Config(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("heads", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
                ("W", ctypes.c_int), ("D", ctypes.c_int), ("topk", ctypes.c_int), ("top_p", ctypes.c_float),
                ("kmin", ctypes.c_int), ("kmax", ctypes.c_int)]


class WorkspaceLayout(ctypes.Structure):
    _fields_ = [(n, ctypes.c_size_t) for n in ("q_cube", "k_cube", "v_cube", "q_pool", "k_pool", "v_pool",
                                               "o_coarse", "s_coarse", "pool_split", "p_split", "cnt", "order",
                                               "err", "total")]


_lib = None


def load():
    """Loads libvsa.so and declares its signatures (no GPU needed)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(lib_path):
        raise RuntimeError(f"{lib_path} is not built; run: python -m trainable_block_sparse_cube_b200.build")
    L = ctypes.CDLL(lib_path)
    vp, i32, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    L.vsa_workspace_bytes.argtypes = [ctypes.POINTER(Config)]
    L.vsa_workspace_bytes.restype = sz
    L.vsa_workspace_layout.argtypes = [ctypes.POINTER(Config), ctypes.POINTER(WorkspaceLayout)]
    L.vsa_workspace_layout.restype = i32
    L.vsa_plan.argtypes = [ctypes.POINTER(vp), ctypes.POINTER(Config), vp, sz]
    L.vsa_plan.restype = i32
    L.vsa_run.argtypes = [vp] * 10
    L.vsa_run.restype = i32
    L.vsa_run_fixed_idx.argtypes = [vp] * 12
    L.vsa_run_host.argtypes = [vp] * 10
    L.vsa_run_host.restype = i32
    L.vsa_run_fixed_idx.restype = i32
    L.vsa_forward.argtypes = [vp] * 5 + [i32] * 7 + [ctypes.c_float, vp, vp, vp]
    L.vsa_forward.restype = i32
    L.vsa_check.argtypes = [vp]
    L.vsa_check.restype = i32
    L.vsa_plan_destroy.argtypes = [vp]
    L.vsa_plan_destroy.restype = None
    L.vsa_status_string.argtypes = [i32]
    L.vsa_status_string.restype = ctypes.c_char_p
    L.vsa_set_wait_limit_ns.argtypes = [vp, ctypes.c_uint64]
    L.vsa_set_wait_limit_ns.restype = i32
    L.vsa_set_debug_stall.argtypes = [vp, i32]
    L.vsa_set_debug_stall.restype = i32
    L.vsa_set_cube_major_copies.argtypes = [vp, i32]
    L.vsa_set_cube_major_copies.restype = i32
    L.vsa_set_stage_timing.argtypes = [vp, i32]
    L.vsa_set_stage_timing.restype = i32
    L.vsa_stage_times.argtypes = [vp, ctypes.POINTER(ctypes.c_float)]
    L.vsa_stage_times.restype = i32
    L.vsa_stage_times_history.argtypes = [vp, ctypes.POINTER(ctypes.c_float), i32, ctypes.POINTER(ctypes.c_int)]
    L.vsa_stage_times_history.restype = i32
    L.vsa_kernels_per_run.argtypes = []
    L.vsa_kernels_per_run.restype = i32
    L.vsa_forward_noalloc.argtypes = [vp] * 5 + [i32] * 7 + [ctypes.c_float, vp, vp, vp]
    L.vsa_forward_noalloc.restype = i32
    L.vsa_run_train.argtypes = [vp] * 12
    L.vsa_run_train.restype = i32
    L.vsa_backward_workspace_bytes.argtypes = [ctypes.POINTER(Config)]
    L.vsa_backward_workspace_bytes.restype = sz
    L.vsa_run_backward.argtypes = [vp, vp, sz] + [vp] * 16
    L.vsa_run_backward.restype = i32
    L.vsa_backward_stage_times.argtypes = [vp, ctypes.POINTER(ctypes.c_float)]
    L.vsa_backward_stage_times.restype = i32
    L.vsa_backward_stage_times_history.argtypes = [vp, ctypes.POINTER(ctypes.c_float), i32, ctypes.POINTER(ctypes.c_int)]
    L.vsa_backward_stage_times_history.restype = i32
    L.vsa_measure_l2_read.argtypes = [vp, sz, i32, vp, vp]
    L.vsa_measure_l2_read.restype = i32
    _lib = L
    return L


def _check(code: int, what: str):
    if code != 0:
        raise VSAError(code, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _need(t, name, dtype, shape):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def make_config(B, heads, T, H, W, D, topk=0, top_p=0.0, kmin=0, kmax=0) -> Config:
    return Config(B, heads, T, H, W, D, topk, top_p, kmin, kmax)


def workspace_bytes(cfg: Config) -> int:
    return int(load().vsa_workspace_bytes(ctypes.byref(cfg)))


def workspace_layout(cfg: Config) -> WorkspaceLayout:
    lay = WorkspaceLayout()
    _check(load().vsa_workspace_layout(ctypes.byref(cfg), ctypes.byref(lay)), "vsa_workspace_layout")
    return lay


class Plan:
    """A plan with its device workspace (a torch uint8 tensor it owns)."""

    def __init__(self, B, heads, T, H, W, D, topk=0, top_p=0.0, kmin=0, kmax=0, device=None):
        L = load()
        self.cfg = make_config(B, heads, T, H, W, D, topk, top_p, kmin, kmax)
        self.B, self.heads, self.T, self.H, self.W, self.D = B, heads, T, H, W, D
        self.N = T * H * W
        self.C = self.N // 64
        self.kcap = topk if topk > 0 else kmax
        nbytes = L.vsa_workspace_bytes(ctypes.byref(self.cfg))
        if nbytes == 0:
            raise VSAError(L.vsa_workspace_layout(ctypes.byref(self.cfg), ctypes.byref(WorkspaceLayout())) or 1,
                           "invalid configuration")
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
        self.workspace = torch.empty(nbytes, dtype=torch.uint8, device=device)
        self.layout = workspace_layout(self.cfg)
        h = ctypes.c_void_p()
        _check(L.vsa_plan(ctypes.byref(h), ctypes.byref(self.cfg), _ptr(self.workspace), nbytes), "vsa_plan")
        self._h = h

    def __del__(self):
        h = getattr(self, "_h", None)
        if h is not None and _lib is not None:
            _lib.vsa_plan_destroy(h)
            self._h = None

    # ------------------------------------------------------------ helpers
    def _inputs(self, q, k, v, gate_c, gate_f):
        BHND = (self.B, self.heads, self.N, self.D)
        for t, n in ((q, "q"), (k, "k"), (v, "v")):
            _need(t, n, torch.bfloat16, BHND)
        for t, n in ((gate_c, "gate_c"), (gate_f, "gate_f")):
            _need(t, n, torch.float32, BHND[:3])

    def run(self, q, k, v, gate_c, gate_f, out=None, idx=None, cnt=None):
        """Whole forward pass. Returns (out, idx, cnt); enqueued on the current stream."""
        self._inputs(q, k, v, gate_c, gate_f)
        dev = q.device
        out = torch.empty_like(q) if out is None else out
        idx = torch.empty((self.B, self.heads, self.C, self.kcap), dtype=torch.int32, device=dev) if idx is None else idx
        cnt = torch.empty((self.B, self.heads, self.C), dtype=torch.int32, device=dev) if cnt is None else cnt
        _check(load().vsa_run(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(gate_c), _ptr(gate_f), _ptr(out), _ptr(idx),
                              _ptr(cnt), _stream()), "vsa_run")
        return out, idx, cnt

    def run_train(self, q, k, v, gate_c, gate_f):
        """Forward pass that also saves the backward pass's inputs. Returns
        (out, idx, cnt, o_fine, lse); enqueued on the current stream."""
        self._inputs(q, k, v, gate_c, gate_f)
        dev = q.device
        out = torch.empty_like(q)
        o_fine = torch.empty(q.shape, dtype=torch.float32, device=dev)
        lse = torch.empty((self.B, self.heads, self.N), dtype=torch.float32, device=dev)
        idx = torch.empty((self.B, self.heads, self.C, self.kcap), dtype=torch.int32, device=dev)
        cnt = torch.empty((self.B, self.heads, self.C), dtype=torch.int32, device=dev)
        _check(load().vsa_run_train(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(gate_c), _ptr(gate_f), _ptr(out),
                                    _ptr(idx), _ptr(cnt), _ptr(o_fine), _ptr(lse), _stream()), "vsa_run_train")
        return out, idx, cnt, o_fine, lse

    def run_backward(self, q, k, v, gate_c, gate_f, idx, cnt, o_fine, lse, dout):
        """Gradients of the gated output with the selection held fixed.
        Returns (dq, dk, dv, dgate_c, dgate_f); enqueued on the current stream.
        The backward workspace is allocated (once) by this plan."""
        self._inputs(q, k, v, gate_c, gate_f)
        BHND = (self.B, self.heads, self.N, self.D)
        _need(idx, "idx", torch.int32, (self.B, self.heads, self.C, self.kcap))
        if cnt is not None:
            _need(cnt, "cnt", torch.int32, (self.B, self.heads, self.C))
        _need(o_fine, "o_fine", torch.float32, BHND)
        _need(lse, "lse", torch.float32, BHND[:3])
        _need(dout, "dout", torch.bfloat16, BHND)
        L = load()
        if getattr(self, "bwd_workspace", None) is None:
            nb = L.vsa_backward_workspace_bytes(ctypes.byref(self.cfg))
            self.bwd_workspace = torch.empty(nb, dtype=torch.uint8, device=q.device)
        dq, dk, dv = torch.empty_like(q), torch.empty_like(q), torch.empty_like(q)
        dgc, dgf = torch.empty_like(gate_c), torch.empty_like(gate_f)
        _check(L.vsa_run_backward(self._h, _ptr(self.bwd_workspace), self.bwd_workspace.numel(), _ptr(q), _ptr(k),
                                  _ptr(v), _ptr(gate_c), _ptr(gate_f), _ptr(idx), _ptr(cnt), _ptr(o_fine), _ptr(lse),
                                  _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dgc), _ptr(dgf), _stream()),
               "vsa_run_backward")
        return dq, dk, dv, dgc, dgf

    def backward_stage_times_history(self, max_runs):
        """[(gather + coarse, prep + lists + coarse backward, dq, dk/dv) ms] of the last timed backward calls."""
        ms = (ctypes.c_float * (4 * max_runs))()
        n = ctypes.c_int(0)
        _check(load().vsa_backward_stage_times_history(self._h, ms, int(max_runs), ctypes.byref(n)),
               "vsa_backward_stage_times_history")
        return [tuple(float(x) for x in ms[4 * i: 4 * i + 4]) for i in range(n.value)]

    def backward_stage_times(self):
        """Device ms of (gather + coarse, prep + lists + coarse backward, dq, dk/dv) of the last timed backward."""
        ms = (ctypes.c_float * 4)()
        _check(load().vsa_backward_stage_times(self._h, ms), "vsa_backward_stage_times")
        return tuple(float(x) for x in ms)

    def run_host(self, q, k, v, gate_c, gate_f, out, idx, cnt=None):
        """Forward pass on host tensors (pinned for overlapped copies): inputs are
        copied in and out/idx/cnt written back by the library; enqueued on the
        current stream (synchronise it before reading the results)."""
        BHND = (self.B, self.heads, self.N, self.D)
        for t, n, dt, sh in ((q, "q", torch.bfloat16, BHND), (k, "k", torch.bfloat16, BHND),
                             (v, "v", torch.bfloat16, BHND), (gate_c, "gate_c", torch.float32, BHND[:3]),
                             (gate_f, "gate_f", torch.float32, BHND[:3]), (out, "out", torch.bfloat16, BHND),
                             (idx, "idx", torch.int32, (self.B, self.heads, self.C, self.kcap)),
                             (cnt, "cnt", torch.int32, (self.B, self.heads, self.C))):
            if t is None and n == "cnt":
                continue
            if not isinstance(t, torch.Tensor) or t.is_cuda or t.dtype != dt or tuple(t.shape) != tuple(sh) \
                    or not t.is_contiguous():
                raise ValueError(f"{n} must be a contiguous host tensor of {dt} and shape {tuple(sh)}")
        _check(load().vsa_run_host(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(gate_c), _ptr(gate_f), _ptr(out),
                                   _ptr(idx), _ptr(cnt), _stream()), "vsa_run_host")
        return out, idx, cnt

    def run_fixed_idx(self, q, k, v, gate_c, gate_f, idx, cnt=None, want_out=True, want_coarse=False,
                      want_fine=False):
        """Forward pass on a given selection. Returns (out, coarse, fine) (None where not requested)."""
        self._inputs(q, k, v, gate_c, gate_f)
        dev = q.device
        _need(idx, "idx", torch.int32, (self.B, self.heads, self.C, self.kcap))
        if cnt is not None:
            _need(cnt, "cnt", torch.int32, (self.B, self.heads, self.C))
        out = torch.empty_like(q) if want_out else None
        oc = torch.empty((self.B, self.heads, self.C, self.D), dtype=torch.float32, device=dev) if want_coarse else None
        of = torch.empty((self.B, self.heads, self.N, self.D), dtype=torch.float32, device=dev) if want_fine else None
        _check(load().vsa_run_fixed_idx(self._h, _ptr(q), _ptr(k), _ptr(v), _ptr(gate_c), _ptr(gate_f), _ptr(idx),
                                        _ptr(cnt), _ptr(out), _ptr(oc), _ptr(of), _stream()), "vsa_run_fixed_idx")
        return out, oc, of

    def check(self):
        """Synchronises and raises VSAError if a device-side error was recorded."""
        _check(load().vsa_check(self._h), "vsa_check")

    def set_wait_limit_ns(self, ns: int):
        _check(load().vsa_set_wait_limit_ns(self._h, int(ns)), "vsa_set_wait_limit_ns")

    def set_debug_stall(self, on: bool):
        _check(load().vsa_set_debug_stall(self._h, 1 if on else 0), "vsa_set_debug_stall")

    def set_cube_major_copies(self, on: bool):
        """Also write the cube-major copy of q into the workspace (k and v are always copied)."""
        _check(load().vsa_set_cube_major_copies(self._h, 1 if on else 0), "vsa_set_cube_major_copies")

    def set_stage_timing(self, on):
        """True (or a run count n >= 1): record stage events of the next runs,
        keeping the last n (1 for True); False/0 switches timing off."""
        n = int(on) if not isinstance(on, bool) else (1 if on else 0)
        _check(load().vsa_set_stage_timing(self._h, n), "vsa_set_stage_timing")

    def stage_times(self):
        """Device ms of (gather+pool, coarse, fine) of the last timed run."""
        ms = (ctypes.c_float * 3)()
        _check(load().vsa_stage_times(self._h, ms), "vsa_stage_times")
        return tuple(float(x) for x in ms)

    def stage_times_history(self, max_runs):
        """[(gather+pool, coarse, fine) ms] of the last timed runs, oldest first."""
        ms = (ctypes.c_float * (3 * max_runs))()
        n = ctypes.c_int(0)
        _check(load().vsa_stage_times_history(self._h, ms, int(max_runs), ctypes.byref(n)), "vsa_stage_times_history")
        return [tuple(float(x) for x in ms[3 * i: 3 * i + 3]) for i in range(n.value)]

    # ------------------------------------------------------------ workspace views
    def workspace_view(self, region: str, dtype, shape):
        off = getattr(self.layout, region)
        nbytes = torch.empty((), dtype=dtype).element_size()
        for s in shape:
            nbytes *= s
        return self.workspace[off: off + nbytes].view(dtype).view(*shape)

    def cube_major(self, which: str):
        return self.workspace_view(f"{which}_cube", torch.bfloat16, (self.B * self.heads, self.C, 64, self.D))

    def pooled(self, which: str):
        return self.workspace_view(f"{which}_pool", torch.float32, (self.B * self.heads, self.C, self.D))


def measure_l2_read(buf, passes, status):
    """Enqueues the L2 -> SM bulk-copy read of the uint8 CUDA tensor `buf`
    (`passes` times) on the current stream; `status` is a zeroed int32 CUDA
    tensor (bit 0 set if a bounded wait gave up)."""
    _need(buf, "buf", torch.uint8, tuple(buf.shape))
    _need(status, "status", torch.int32, tuple(status.shape))
    _check(load().vsa_measure_l2_read(_ptr(buf), buf.numel(), int(passes), _ptr(status), _stream()),
           "vsa_measure_l2_read")


def forward(q, k, v, gate_c, gate_f, T, H, W, topk=0, top_p=0.0, out=None, idx=None):
    """One-call form (library-owned plan cache). Returns (out, idx)."""
    B, heads, N, D = q.shape
    if N != T * H * W:
        raise ValueError("N must equal T*H*W")
    C = N // 64
    kcap = topk if topk > 0 else min(128, C)
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _need(t, n, torch.bfloat16, (B, heads, N, D))
    for t, n in ((gate_c, "gate_c"), (gate_f, "gate_f")):
        _need(t, n, torch.float32, (B, heads, N))
    out = torch.empty_like(q) if out is None else out
    idx = torch.empty((B, heads, C, kcap), dtype=torch.int32, device=q.device) if idx is None else idx
    _check(load().vsa_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(gate_c), _ptr(gate_f), B, heads, T, H, W, D, topk,
                              ctypes.c_float(top_p), _ptr(out), _ptr(idx), _stream()), "vsa_forward")
    return out, idx
