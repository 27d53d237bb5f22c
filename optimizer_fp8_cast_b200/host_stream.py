"""Training steps on inputs that live in host memory, with the transfers overlapped.

A caller whose X and dY arrive in (pinned) host memory and who needs Y and dX back on the host
pays two PCIe transfers per step. Run back to back, copy in -> step -> copy out, the step time is
their sum. HostStreamedStep keeps three CUDA streams busy at once:

  copy-in stream   X, dY of step t+1 -> device buffer set (t+1) % 2
  compute stream   step t on buffer set t % 2 (the library's kernels)
  copy-out stream  Y, dX of step t-1 -> host

so a step costs about the slower of the two copy directions (the copy engines run in both
directions at once). Ordering is kept with CUDA events only: a buffer set is refilled only after
the step that read it has finished, and its outputs are overwritten only after they were copied
out. Nothing synchronises with the host until `finish()`.
"""
import torch


class HostStreamedStep:
    def __init__(self, step):
        """step: an Fp8LinearStep. Allocates two device sets of X, dY, Y and dX per layer."""
        self.st = step
        dev = step.device
        bf = dict(dtype=torch.bfloat16, device=dev)
        T = step.tokens
        self.x = [[torch.empty(T, L.fin, **bf) for L in step.layers] for _ in range(2)]
        self.dy = [[torch.empty(T, L.fout, **bf) for L in step.layers] for _ in range(2)]
        self.y = [[torch.empty(T, L.fout, **bf) for L in step.layers] for _ in range(2)]
        self.dx = [[torch.empty(T, L.fin, **bf) for L in step.layers] for _ in range(2)]
        self.s_in = torch.cuda.Stream(device=dev)
        self.s_compute = torch.cuda.Stream(device=dev)
        self.s_out = torch.cuda.Stream(device=dev)
        self.copied_in = [torch.cuda.Event() for _ in range(2)]
        self.computed = [torch.cuda.Event() for _ in range(2)]
        self.copied_out = [torch.cuda.Event() for _ in range(2)]
        self.used = [False, False]
        self.n = 0

    def step(self, xs_host, dys_host, ys_host, dxs_host):
        """Enqueue one step: inputs from host tensors xs_host / dys_host (one per layer, pinned
        for asynchronous copies), outputs into host tensors ys_host / dxs_host."""
        b = self.n % 2
        st = self.st
        with torch.cuda.stream(self.s_in):
            if self.used[b]:
                self.s_in.wait_event(self.computed[b])        # step n-2 has read set b
            for dst, src in zip(self.x[b], xs_host):
                dst.copy_(src, non_blocking=True)
            for dst, src in zip(self.dy[b], dys_host):
                dst.copy_(src, non_blocking=True)
            self.copied_in[b].record(self.s_in)
        with torch.cuda.stream(self.s_compute):
            self.s_compute.wait_event(self.copied_in[b])
            if self.used[b]:
                self.s_compute.wait_event(self.copied_out[b])  # outputs of step n-2 are out
            for k, L in enumerate(st.layers):
                L.Y, L.dX = self.y[b][k], self.dx[b][k]
            st.step(self.x[b], self.dy[b])
            self.computed[b].record(self.s_compute)
        with torch.cuda.stream(self.s_out):
            self.s_out.wait_event(self.computed[b])
            for dst, src in zip(ys_host, self.y[b]):
                dst.copy_(src, non_blocking=True)
            for dst, src in zip(dxs_host, self.dx[b]):
                dst.copy_(src, non_blocking=True)
            self.copied_out[b].record(self.s_out)
        self.used[b] = True
        self.n += 1

    def finish(self):
        """Wait for every enqueued step and copy."""
        for s in (self.s_in, self.s_compute, self.s_out):
            s.synchronize()
