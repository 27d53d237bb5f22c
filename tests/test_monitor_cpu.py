"""Host-side health monitor logic (no GPU): skip on a non-finite norm, amax spikes against the
mean of the previous checks ("FP8 混合精度训练工程实践" §七: 3x the mean of the last checks)."""
from optimizer_fp8_cast_b200.monitor import HealthMonitor


def test_spike_needs_a_full_window_and_three_times_the_mean():
    m = HealthMonitor(n_tensors=2, window=9, spike_ratio=3.0)
    for s in range(9):
        assert m.check(s, [1.0, 2.0], 0.5, 0) == []
    ev = m.check(9, [3.5, 5.9], 0.5, 0)
    assert [e[0] for e in ev] == ["amax_spike"] and "tensor 0" in ev[0][2]   # 3.5 > 3 x 1.0
    # tensor 1's window is now eight 2.0 and one 5.9 (3 x mean = 7.3): 7.2 passes; then the
    # window is seven 2.0, 5.9 and 7.2 (3 x mean = 9.033...): 9.1 flags
    assert m.check(10, [1.0, 7.2], 0.5, 0) == []
    ev = m.check(11, [1.0, 9.1], 0.5, 0)
    assert [e[0] for e in ev] == ["amax_spike"] and "tensor 1" in ev[0][2]


def test_first_checks_never_flag_and_zero_mean_is_ignored():
    m = HealthMonitor(n_tensors=1, window=3)
    assert m.check(0, [0.0], 1.0, 0) == [] and m.check(1, [0.0], 1.0, 0) == []
    assert m.check(2, [0.0], 1.0, 0) == [] and m.check(3, [100.0], 1.0, 0) == []


def test_nonfinite_norm_and_amax():
    m = HealthMonitor(n_tensors=2)
    kinds = [e[0] for e in m.check(5, [float("nan"), 1.0], float("inf"), 1)]
    assert kinds == ["skip", "nonfinite_amax"]
    kinds = [e[0] for e in m.check(6, [1.0, 1.0], 0.2, 0, counters=[[0, 0, 3], [0, 0, 0]], numel=[10, 10])]
    assert kinds == ["nonfinite_input"]


def test_state_dict_round_trips_through_torch_save():
    """The training state of a step object (built on the CPU: no kernel runs) survives
    torch.save / torch.load and restores into a fresh object."""
    import io
    import torch
    from optimizer_fp8_cast_b200.step import Fp8LinearStep
    hp = dict(lr=1e-3, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, loss_scale=1.0,
              max_grad_norm=1.0)
    g = torch.Generator().manual_seed(3)
    w = [torch.randn(64, 32, generator=g)]
    a = Fp8LinearStep([(64, 32)], 16, 4, adamw=hp, w_init=w, device="cpu", device_step=True)
    a.t = 7
    a.history.uniform_(generator=g); a.scale.uniform_(generator=g); a.scale_inv.uniform_(generator=g)
    a.layers[0].m.uniform_(generator=g); a.layers[0].v.uniform_(generator=g)
    a.step_counter.fill_(7)
    buf = io.BytesIO()
    torch.save(a.state_dict(), buf)
    buf.seek(0)
    b = Fp8LinearStep([(64, 32)], 16, 4, adamw=hp, w_init=[torch.zeros(64, 32)], device="cpu",
                      device_step=True)
    b.load_state_dict(torch.load(buf))
    assert b.t == 7 and int(b.step_counter) == 7
    for name in ("history", "scale", "scale_inv", "amax"):
        assert torch.equal(getattr(a, name), getattr(b, name))
    for name in ("W", "master", "m", "v"):
        assert torch.equal(getattr(a.layers[0], name), getattr(b.layers[0], name))
