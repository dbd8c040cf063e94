"""Host-side behaviour of the Python binding (CPU, no GPU needed).

The binding only marshals arguments: with the library missing it must fail
loudly (there is no CPU fallback), and tensors of the wrong device, dtype,
shape or layout must be rejected before anything reaches the library.
"""
import pytest
import torch

from trainable_block_sparse_cube_b200 import synth, vsa


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(vsa, "lib_path", str(tmp_path / "libvsa.so"))
    monkeypatch.setattr(vsa, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        vsa.load()


def test_need_rejects_host_tensors():
    wl = synth.WORKLOADS["tiny"]
    q = synth.make_inputs(wl)[0]
    with pytest.raises(ValueError, match="CUDA tensor"):
        vsa._need(q, "q", torch.bfloat16, (wl.B, wl.heads, wl.N, wl.D))


class _FakeCuda(torch.Tensor):
    """A CPU tensor that claims to live on the GPU, to reach the dtype, shape
    and layout checks of the binding without a device."""

    @property
    def is_cuda(self):
        return True


def _fake(t):
    return t.as_subclass(_FakeCuda)


def test_need_checks_dtype_shape_and_contiguity():
    wl = synth.WORKLOADS["tiny"]
    q = _fake(synth.make_inputs(wl)[0])
    shape = (wl.B, wl.heads, wl.N, wl.D)
    vsa._need(q, "q", torch.bfloat16, shape)  # accepted
    with pytest.raises(ValueError, match="must be torch.float32"):
        vsa._need(q, "gate_c", torch.float32, shape)
    with pytest.raises(ValueError, match="shape"):
        vsa._need(q, "q", torch.bfloat16, (wl.B, wl.heads, wl.N, wl.D + 1))
    with pytest.raises(ValueError, match="contiguous"):
        vsa._need(_fake(q.transpose(2, 3).contiguous().transpose(2, 3)), "q", torch.bfloat16, shape)


def test_run_host_rejects_device_or_mismatched_tensors():
    """run_host validates before calling the library (the plan handle is never used)."""
    wl = synth.WORKLOADS["tiny"]
    q, k, v, gc, gf = synth.make_inputs(wl)
    plan = vsa.Plan.__new__(vsa.Plan)  # no workspace: the checks come first
    plan.B, plan.heads, plan.N, plan.D, plan.C, plan.kcap = wl.B, wl.heads, wl.N, wl.D, wl.C, wl.kcap
    plan._h = None
    out = torch.empty_like(q)
    idx = torch.empty((wl.B, wl.heads, wl.C, wl.kcap), dtype=torch.int32)
    with pytest.raises(ValueError, match="gate_c"):
        plan.run_host(q, k, v, gc.double(), gf, out, idx)
    with pytest.raises(ValueError, match="idx"):
        plan.run_host(q, k, v, gc, gf, out, idx[..., :1])
    with pytest.raises(ValueError, match="q"):
        plan.run_host(_fake(q), k, v, gc, gf, out, idx)
