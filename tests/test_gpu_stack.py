"""Teacher-forced parity of the decode stack against the oracle.

tpl_decode_stack chains the layers on the device: the down projection of
layer l writes layer l+1's input and its normalised operand, and the layers
are launched back to back.  Here the stack's own input to a layer is
captured by running the stack truncated to that many layers (a plan with
n_layers = l whose y is layer l-1's output), the oracle evaluates layer l on
exactly those bits with layer l's weights and cache, and the full stack's
output of layer l (the stack truncated to l+1 layers) must match it element
by element at the 2e-2 tolerance.  The pages' stack is 2L reductions
per forward pass ("Tensor parallel scaling curves", "What tensor parallelism
actually splits"); each truncated run is checked to count 2 per layer.
"""
import numpy as np
import pytest

from tests.conftest import has_gpu

pytestmark = pytest.mark.gpu

if has_gpu():
    import torch

    import oracle
    from megatron_tensor_transformer_plan_b200 import synth, tpl
    from tests.gpu_util import TOL, assert_close_rel, to_np


class Stack:
    """Seeded layers as the benchmark builds them: per-layer weights packed
    for t shards and a cache generated directly in the packed layout
    [t][B][n_kv/t][S+1][d]."""

    def __init__(self, H, nq, nkv, d, F, t, B, S, NL, seed=0, gamma_std=0.0, device="cuda"):
        self.H, self.nq, self.nkv, self.d, self.F, self.t, self.B, self.S, self.NL = H, nq, nkv, d, F, t, B, S, NL
        self.seed, self.gamma_std, self.device = seed, gamma_std, device
        self.flags = tpl.TPL_NORM | tpl.TPL_RESIDUAL
        plan = self.plan(NL)
        self.packed, self.kv, self.keep = [], [], []
        for l in range(NL):
            w = self.weights(l)
            self.packed.append(plan.pack_layer(w))
            del w
            k, v = synth.kv_cache((t, B, nkv // t, S + 1, d), seed=seed, layer=l, device=device)
            self.keep.append((k, v))
            self.kv.append(tpl.Plan.kv(k, v, B, S + 1))
        self.x = synth.activations(B, H, seed=seed, dtype=torch.bfloat16, device=device)
        torch.cuda.synchronize()

    def plan(self, n_layers):
        return tpl.Plan(tpl.make_dims(self.H, self.nq, self.nkv, self.d, self.F, n_layers, 1e-5, self.flags), self.t)

    def weights(self, l):
        return synth.layer_weights(self.H, self.nq, self.nkv, self.d, self.F, seed=self.seed, layer=l,
                                   dtype=torch.bfloat16, device=self.device, gamma_std=self.gamma_std)

    def run(self, n_layers, mode=None):
        """The first n_layers layers as one stack call: (y bf16, y32 fp32)."""
        mode = tpl.TPL_REDUCE_FUSED if mode is None else mode
        plan = self.plan(n_layers)
        ws = plan.workspace(self.B, self.S, device=self.device)
        y = torch.empty_like(self.x)
        y32 = torch.empty((self.B, self.H), dtype=torch.float32, device=self.device)
        plan.reset_counters()
        plan.decode_stack(self.packed[:n_layers], self.kv[:n_layers], self.x, self.S, y, y32, ws, mode)
        torch.cuda.synchronize()
        assert plan.last_device_error() == tpl.TPL_OK
        assert plan.reduction_count() == 2 * n_layers
        return y, y32

    def layer_input(self, l):
        return self.x if l == 0 else self.run(l)[0]

    def oracle_layer(self, l, x):
        """The oracle's layer l on the given input bits and layer l's cache
        (logical layout [B][n_kv][S+1][d], kv head j = s*n_kv/t + local)."""
        w = self.weights(l)
        wb = {k: synth.bits(v) for k, v in w.items()}
        del w
        k, v = self.keep[l]
        t, B, nkv, d = self.t, self.B, self.nkv, self.d

        def logical(c):
            return c.view(t, B, nkv // t, self.S + 1, d).permute(1, 0, 2, 3, 4).reshape(B, nkv, self.S + 1, d)

        od = oracle.Dims(self.H, self.nq, self.nkv, self.d, self.F, eps=1e-5, flags=oracle.NORM | oracle.RESIDUAL)
        y, _ = oracle.decode_layer(od, wb, to_np(x), synth.bits(logical(k)), synth.bits(logical(v)), self.S,
                                   trace=True)
        return y


def _check_layers(st, layers, mode=None):
    worst = {}
    for l in layers:
        x_l = st.layer_input(l)
        y_l, y32_l = st.run(l + 1, mode)
        ref = st.oracle_layer(l, x_l)
        worst[l] = assert_close_rel(to_np(y32_l), ref, tol=TOL, what=f"layer {l} y32 (teacher-forced)")
        assert_close_rel(to_np(y_l), ref, tol=TOL, what=f"layer {l} y (teacher-forced)")
    return worst


def test_stack_teacher_forced_small_every_layer(gpu):
    """Five small layers with non-unit gains, 3 tokens (the mma.sync
    projections on layers this small), every layer against the oracle; fused
    and separate stacks equal bit for bit."""
    st = Stack(512, 8, 4, 128, 1024, 4, 3, 50, 5, seed=9, gamma_std=0.02, device=gpu)
    _check_layers(st, range(5))
    ys, ys32 = st.run(5, tpl.TPL_REDUCE_SEPARATE)
    yf, yf32 = st.run(5)
    assert torch.equal(ys32, yf32) and torch.equal(ys, yf)


def test_stack_teacher_forced_small_tc_family(gpu):
    """Four small layers with non-unit gains at 16 tokens, where the
    tensor-core projections run on any layer size and every layer's QKV
    operand comes from the previous layer's down epilogue (so it must carry
    the next layer's gain)."""
    st = Stack(1024, 16, 8, 128, 2816, 8, 16, 100, 4, seed=10, gamma_std=0.02, device=gpu)
    assert st.plan(4).decode_kernel_count(16, n_layers=4) == 5 * 4 + 1
    _check_layers(st, range(4))


@pytest.mark.slow
def test_stack_70b_teacher_forced_layers_0_39_79(gpu):
    """The benchmark's workload: 80 70B-shaped layers in the t = 8 layout,
    batch 4, KV length 4096, seed 0, the default kernel choice (tensor-core
    projections at 4 tokens on these layers).  Layers 0, 39 and 79 are
    checked against the oracle on the inputs the stack gave them."""
    torch.cuda.empty_cache()
    free, _ = torch.cuda.mem_get_info()
    assert free > 150e9, f"the 80-layer stack needs about 143 GB of device memory; {free / 1e9:.1f} GB free"
    H, nq, nkv, d, F, t, B, S, NL = 8192, 64, 8, 128, 28672, 8, 4, 4096, 80
    st = Stack(H, nq, nkv, d, F, t, B, S, NL, seed=0, device=gpu)
    try:
        assert st.plan(NL).decode_kernel_count(B, n_layers=NL) == 5 * NL + 1  # the tensor-core family
        worst = _check_layers(st, (0, 39, 79))
        print("teacher-forced worst normalised errors:", worst)
    finally:
        del st
        torch.cuda.empty_cache()
