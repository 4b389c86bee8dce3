"""GPU parity of the prefill layer (tcgen05 projections, causal attention)
against the oracle's unsharded prefill, element by element on the same seeded
inputs.  Tolerance as for decode: |gpu - oracle| <= 2e-2 * (|oracle| +
RMS(oracle)); the fused and separate row-split sums must agree bit for bit."""
import numpy as np
import pytest
import torch

from tests.conftest import has_gpu

pytestmark = pytest.mark.gpu

if has_gpu():
    import oracle
    from megatron_tensor_transformer_plan_b200 import synth, tpl
    from tests.gpu_util import assert_close_rel, to_np

SENTINEL = 0x3F80  # bf16 1.0: cache slots past the chunk must keep it


class Prefill:
    def __init__(self, H, nq, nkv, F, t, T, *, seed=0, layer=0, gamma_std=0.0, S_cap=None,
                 flags=None, attn_mode=0):
        flags = tpl.TPL_NORM | tpl.TPL_RESIDUAL if flags is None else flags
        self.dims = tpl.make_dims(H, nq, nkv, 128, F, 1, 1e-5, flags)
        self.plan = tpl.Plan(self.dims, t)
        self.plan.set_option(tpl.TPL_OPT_PREFILL_ATTN, attn_mode)
        self.t, self.T = t, T
        self.S_cap = S_cap or T + 5
        self.w = synth.layer_weights(H, nq, nkv, 128, F, seed=seed, layer=layer, dtype=torch.bfloat16,
                                     device="cuda", gamma_std=gamma_std)
        self.packed = self.plan.pack_layer(self.w)
        self.x = synth.activations(T, H, seed=seed, layer=layer, dtype=torch.bfloat16, device="cuda")
        n = nkv * self.S_cap * 128
        self.k = torch.full((n,), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        self.v = torch.full((n,), SENTINEL, dtype=torch.int16, device="cuda").view(torch.bfloat16)
        self.kv = tpl.Plan.kv(self.k, self.v, 1, self.S_cap)
        self.ws = self.plan.prefill_workspace(T)
        torch.cuda.synchronize()

    def run(self, mode=None):
        mode = tpl.TPL_REDUCE_FUSED if mode is None else mode
        y = torch.empty_like(self.x)
        y32 = torch.empty(self.x.shape, dtype=torch.float32, device="cuda")
        self.plan.prefill_layer(self.packed, self.kv, self.x, y, y32, self.ws, mode)
        torch.cuda.synchronize()
        return y, y32

    def intermediates(self):
        d, T = self.dims, self.T
        off = self.plan.prefill_intermediates(T)
        nqd = d.n_q_heads * d.head_dim

        def view(o, n, dt):
            nb = n * torch.tensor([], dtype=dt).element_size()
            return self.ws[o:o + nb].view(dt)

        o_hi = view(off["o"], T * nqd, torch.bfloat16).view(T, nqd)
        o_lo = view(off["o_lo"], T * nqd, torch.bfloat16).view(T, nqd)
        return {"q": view(off["q"], T * nqd, torch.float32).view(T, nqd),
                "attn_hi": o_hi,
                "attn": o_hi.float() + o_lo.float(),
                "h": view(off["h"], T * d.hidden, torch.float32).view(T, d.hidden),
                "act": view(off["act"], T * d.ffn, torch.bfloat16).view(T, d.ffn)}

    def cache(self):
        """Cache slots 0..T-1 gathered back to [T][n_kv*d], and the slots past T."""
        d, t = self.dims, self.t
        nkv_s = d.n_kv_heads // t
        kk = self.k.view(t, 1, nkv_s, self.S_cap, 128)[:, 0]  # [t][nkv_s][S_cap][d]
        vv = self.v.view(t, 1, nkv_s, self.S_cap, 128)[:, 0]
        kt = kk[:, :, :self.T].permute(2, 0, 1, 3).reshape(self.T, -1)
        vt = vv[:, :, :self.T].permute(2, 0, 1, 3).reshape(self.T, -1)
        rest = torch.cat([kk[:, :, self.T:].reshape(-1), vv[:, :, self.T:].reshape(-1)])
        return kt, vt, rest

    def _oracle_args(self):
        d = self.dims
        dims = oracle.Dims(d.hidden, d.n_q_heads, d.n_kv_heads, d.head_dim, d.ffn, eps=float(d.rms_eps),
                           flags=int(d.flags) & (tpl.TPL_NORM | tpl.TPL_RESIDUAL | tpl.TPL_ROPE),
                           rope_base=float(d.rope_base))
        w = {k: synth.bits(v) for k, v in self.w.items()}
        return dims, w, to_np(self.x)

    def oracle(self):
        return oracle.prefill_layer(*self._oracle_args(), trace=True)

    def oracle_rows(self, rows):
        return oracle.prefill_rows(*self._oracle_args(), rows, trace=True)


def check_prefill(P: Prefill):
    y, y32 = P.run(tpl.TPL_REDUCE_FUSED)
    inter = {k: v.clone() for k, v in P.intermediates().items()}
    ref_y, ref_k, ref_v, tr = P.oracle()
    assert_close_rel(to_np(inter["q"]), tr["q"], what="q")
    kt, vt, rest = P.cache()
    assert_close_rel(to_np(kt), ref_k, what="k (cache slots 0..T-1)")
    assert_close_rel(to_np(vt), ref_v, what="v (cache slots 0..T-1)")
    assert bool((rest.view(torch.int16) == SENTINEL).all()), "cache slots past the chunk were written"
    assert_close_rel(to_np(inter["attn"]), tr["attn"], what="attention output")
    assert_close_rel(to_np(inter["h"]), tr["h"], what="h")
    assert_close_rel(to_np(inter["act"]), tr["act"], what="act")
    assert_close_rel(to_np(y32), ref_y, what="y32")
    assert_close_rel(to_np(y), ref_y, what="y")
    assert torch.equal(y, y32.bfloat16())
    ys, ys32 = P.run(tpl.TPL_REDUCE_SEPARATE)
    assert torch.equal(ys32, y32), "fused and separate reductions differ"
    assert torch.equal(ys, y)
    assert P.plan.last_device_error() == tpl.TPL_OK


SMALL = [
    # H, nq, nkv, F, t, T
    (1024, 16, 4, 2816, 4, 200),   # two 128-token tiles (ragged), 4 TMEM accumulators
    (1024, 16, 8, 2816, 8, 130),   # t = 8: F/t = 352, K tiles cross shard boundaries
    (512, 8, 2, 1376, 2, 77),      # t = 2, F/t = 688
    (768, 12, 4, 1056, 1, 33),     # t = 1, 2F = 2112: ragged 256-column tile, g = 3
    (512, 16, 1, 512, 1, 64),      # g = 16: two head chunks per kv head
    (520, 4, 2, 704, 2, 50),       # hidden = 520: ragged 16-column epilogue chunk
    (256, 2, 2, 256, 2, 1),        # one token
]


@pytest.mark.parametrize("case", SMALL)
def test_prefill_small(gpu, case):
    H, nq, nkv, F, t, T = case
    check_prefill(Prefill(H, nq, nkv, F, t, T, gamma_std=0.02 if T > 100 else 0.0))


def tile_waves(M, N, shards=1, sms=148):
    """Output tiles of one prefill GEMM (128 x 256) and how many of them the
    kernel runs as half tiles on `sms` SMs: the partial last wave, when it
    fills at most half of them."""
    tiles = -(-M // 128) * -(-N // 256) * shards
    rem = tiles % sms
    return tiles, (rem if 0 < rem and 2 * rem <= sms else 0)


@pytest.mark.parametrize("flags", ["default", "rope"])
def test_prefill_half_tiles_change_no_bits(gpu, flags):
    """The half tiles of a partial last wave (N = 128 products over the same
    K steps in the same order) give the same bits as whole tiles, for every
    output of the layer, in both reduction modes."""
    H, nq, nkv, F, t, T = 1024, 16, 8, 2816, 4, 1280
    fl = None if flags == "default" else tpl.TPL_NORM | tpl.TPL_RESIDUAL | tpl.TPL_ROPE
    P = Prefill(H, nq, nkv, F, t, T, seed=5, flags=fl)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    rps = (nq // t + 2 * (nkv // t)) * 128
    # QKV 160 tiles (12 as halves), gate/up 220 (72), O and down fused 40 (all
    # halves), separate 160 (12): both kinds of unit in every kernel family
    waves = [tile_waves(T, t * rps, 1, sms), tile_waves(T, 2 * F, 1, sms), tile_waves(T, H, 1, sms),
             tile_waves(T, H, t, sms)]
    assert all(h > 0 for _, h in waves), waves
    assert any(tiles > h for tiles, h in waves), waves

    def outputs():
        out = {}
        for mode in (tpl.TPL_REDUCE_FUSED, tpl.TPL_REDUCE_SEPARATE):
            y, y32 = P.run(mode)
            out[f"y{mode}"], out[f"y32_{mode}"] = y, y32
            out.update({f"{k}{mode}": v.clone() for k, v in P.intermediates().items()})
            kt, vt, _ = P.cache()
            out[f"k{mode}"], out[f"v{mode}"] = kt.clone(), vt.clone()
        return out

    P.plan.set_option(tpl.TPL_OPT_PREFILL_TAIL, 1)
    halves = outputs()
    P.plan.set_option(tpl.TPL_OPT_PREFILL_TAIL, 0)
    whole = outputs()
    for k in halves:
        assert torch.equal(halves[k].view(torch.uint8), whole[k].view(torch.uint8)), k
    assert P.plan.last_device_error() == tpl.TPL_OK


@pytest.mark.parametrize("case", [(1024, 16, 4, 2816, 4, 200), (512, 16, 1, 512, 1, 64)])
def test_prefill_mma_sync_attention(gpu, case):
    """The mma.sync attention kernel (kept to measure against) on group sizes
    the tensor-core kernel also takes."""
    H, nq, nkv, F, t, T = case
    check_prefill(Prefill(H, nq, nkv, F, t, T, attn_mode=1))


def test_prefill_attention_kernels_agree(gpu):
    """Both attention kernels against each other on the same chunk."""
    outs = []
    for mode in (0, 1):
        P = Prefill(1024, 16, 2, 1408, 2, 300, attn_mode=mode)
        P.run()
        outs.append(P.intermediates()["attn"].clone())
    assert_close_rel(to_np(outs[0]), to_np(outs[1]).astype(np.float64), tol=2e-3, what="tcgen05 vs mma.sync")


def test_prefill_first_token_is_decode_of_empty_cache(gpu):
    """Token 0 of a prefill sees only itself: its attention output equals its
    own v (to bf16 rounding), as in a decode step with S = 0."""
    P = Prefill(1024, 16, 4, 2816, 4, 40)
    P.run()
    inter = P.intermediates()
    kt, vt, _ = P.cache()
    g = 4
    v0 = vt[0].view(4, 128).float()
    a0 = inter["attn"][0].view(16, 128)
    expect = v0.repeat_interleave(g, dim=0)
    # the only key's weight is exactly 1, so the output is v itself (hi + lo);
    # the cache holds rn(v), at most half a bf16 step away
    assert bool(((a0 - expect).abs() <= expect.abs() * 2.0**-8).all())


def test_prefill_rejects(gpu):
    P = Prefill(512, 8, 2, 1376, 2, 16)
    y, y32 = P.run()
    small = P.ws[: P.ws.numel() - 256]
    with pytest.raises(tpl.TplError) as e:
        P.plan.prefill_layer(P.packed, P.kv, P.x, y, y32, small, tpl.TPL_REDUCE_FUSED)
    assert e.value.code == tpl.TPL_EWORKSPACE
    kv_short = tpl.Plan.kv(P.k, P.v, 1, 15)
    with pytest.raises(tpl.TplError) as e:
        P.plan.prefill_layer(P.packed, kv_short, P.x, y, y32, P.ws, tpl.TPL_REDUCE_FUSED)
    assert e.value.code == tpl.TPL_ENOMEM


@pytest.mark.slow
def test_prefill_long_chunk_small_dims(gpu):
    """T = 2048 (the chunk length of the 70B prefill workload) at small dims."""
    check_prefill(Prefill(1024, 16, 8, 2816, 8, 2048, gamma_std=0.02))


@pytest.mark.slow
def test_prefill_70b_dims_short_chunk(gpu):
    """The 70B layer's dimensions (t = 8) over a short ragged chunk."""
    check_prefill(Prefill(8192, 64, 8, 28672, 8, 40))


@pytest.mark.slow
def test_prefill_70b_chunk_2048_sampled_rows(gpu):
    """The 70B prefill workload at full size (t = 8, 2048 tokens): every
    key/value the chunk writes, and the layer's outputs and intermediates at
    sampled tokens (both ends of the chunk, either side of a 128-token tile
    edge, the middle), against the oracle computed row by row."""
    P = Prefill(8192, 64, 8, 28672, 8, 2048, S_cap=2048 + 64)
    y, y32 = P.run(tpl.TPL_REDUCE_FUSED)
    inter = {k: v.clone() for k, v in P.intermediates().items()}
    rows = [0, 1, 127, 128, 1000, 2047]
    ref_y, ref_k, ref_v, tr = P.oracle_rows(rows)
    kt, vt, rest = P.cache()
    assert_close_rel(to_np(kt), ref_k, what="k (all 2048 cache slots)")
    assert_close_rel(to_np(vt), ref_v, what="v (all 2048 cache slots)")
    assert bool((rest.view(torch.int16) == SENTINEL).all())
    assert_close_rel(to_np(inter["q"][rows]), tr["q"], what="q")
    assert_close_rel(to_np(inter["attn"][rows]), tr["attn"], what="attention output")
    assert_close_rel(to_np(inter["h"][rows]), tr["h"], what="h")
    assert_close_rel(to_np(inter["act"][rows]), tr["act"], what="act")
    assert_close_rel(to_np(y32[rows]), ref_y, what="y32")
    assert_close_rel(to_np(y[rows]), ref_y, what="y")
    ys, ys32 = P.run(tpl.TPL_REDUCE_SEPARATE)
    assert torch.equal(ys32, y32), "fused and separate reductions differ"
    assert P.plan.last_device_error() == tpl.TPL_OK
