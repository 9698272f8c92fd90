"""Host logic of the torch front end, on CPU: the plan cache.

A plan's workspace serves one call at a time, so the cache keeps one plan per
(shape, device, stream); calls on one stream run in order and may share it.
Plan construction (which allocates device memory) is replaced by a stub here.
"""
import selective_state_space_30_b200 as ssm


class _StubPlan:
    made = 0

    def __init__(self, *args):
        _StubPlan.made += 1
        self.args = args


class _TorchLikeStream:
    def __init__(self, handle):
        self.cuda_stream = handle


def test_one_plan_per_shape_device_and_stream(monkeypatch):
    monkeypatch.setattr(ssm, "Plan", _StubPlan)
    monkeypatch.setattr(ssm, "_plans", {})
    shape = (2, 64, 128, 16, 0, 1, ssm.SSM_BF16)
    a = ssm.get_plan(*shape, device=0, stream=0x1000)
    assert ssm.get_plan(*shape, device=0, stream=0x1000) is a                       # same stream: shared
    assert ssm.get_plan(*shape, device=0, stream=_TorchLikeStream(0x1000)) is a     # a stream object, same handle
    assert ssm.get_plan(*shape, device=0, stream=0x2000) is not a                   # another stream
    assert ssm.get_plan(*shape, device=1, stream=0x1000) is not a                   # another device
    assert ssm.get_plan(2, 64, 256, 16, 0, 1, ssm.SSM_BF16, device=0, stream=0x1000) is not a   # another shape
    # the legacy default stream: None and 0 name the same one
    assert ssm.get_plan(*shape, device=0, stream=None) is ssm.get_plan(*shape, device=0, stream=0)
    # nheads 0 and nheads == dim are the same (per-channel) layout
    assert ssm.get_plan(2, 64, 128, 16, 64, 1, ssm.SSM_BF16, device=0, stream=0x1000) is a
    assert _StubPlan.made == 5
