"""Host-side health monitor of the FP8 scale state and the gradient norm.

Follows the checks of "FP8 混合精度训练工程实践" §七 (numeric health: NaN/Inf in the gradients
means skip the batch; an amax more than 3x the mean of the recent checks is a spike worth a
warning; check every N steps) and the per-layer metrics of "LLM FP8 微调上线生产实战" 第四步
(amax, scale, saturation and zero fractions). It only reads device buffers the step already
fills (amax history entry 0, scales, the global norm, the skip flag, the optional counters), so
it adds no work to the step; reading them synchronises with the device, which is why it runs
every `every` steps.
"""
from collections import deque


class HealthMonitor:
    def __init__(self, n_tensors, every=100, window=9, spike_ratio=3.0):
        self.every = every
        self.window = window
        self.spike_ratio = spike_ratio
        self.recent = [deque(maxlen=window) for _ in range(n_tensors)]
        self.events = []

    def check(self, step, amax, grad_norm, skipped, scale=None, counters=None, numel=None):
        """Record one check from host values: amax [n] (the newest history entries), the global
        norm and skip flag of the last AdamW call, optionally scales [n] and counters [n][3]
        with the element counts [n]. Returns the list of events raised by this check."""
        ev = []
        if skipped or grad_norm != grad_norm or grad_norm in (float("inf"), float("-inf")):
            ev.append(("skip", step, "non-finite gradient norm: the update was skipped"))
        for i, a in enumerate(amax):
            if a != a or a in (float("inf"), float("-inf")):
                ev.append(("nonfinite_amax", step, f"tensor {i}: amax {a}"))
                continue
            hist = self.recent[i]
            if len(hist) == self.window:
                mean = sum(hist) / len(hist)
                if mean > 0 and a > self.spike_ratio * mean:
                    ev.append(("amax_spike", step,
                               f"tensor {i}: amax {a:.4g} > {self.spike_ratio:g} x recent mean {mean:.4g}"))
            hist.append(a)
        if counters is not None and numel is not None:
            for i, (c, n) in enumerate(zip(counters, numel)):
                if c[2]:
                    ev.append(("nonfinite_input", step, f"tensor {i}: {int(c[2])} NaN/Inf inputs"))
        self.events += ev
        return ev

    def maybe_check(self, st):
        """Every `every` steps of an Fp8LinearStep: read its buffers and check them."""
        if st.t % self.every:
            return []
        amax = st.history[:, 0].tolist()
        return self.check(st.t, amax, float(st.grad_norm.item()), int(st.skipped.item()),
                          scale=st.scale.tolist(),
                          counters=st.counters.tolist() if st.counters is not None else None,
                          numel=None)
