"""GPU parity of the rotary position embedding (TPL_ROPE) in decode and in
prefill, and of chunked prefill into a cache that already holds earlier
tokens (tpl_prefill_chunk), against the oracle on the same seeded inputs.
Tolerance as everywhere: |gpu - oracle| <= 2e-2 * (|oracle| + RMS(oracle))
per element; the fused and separate row-split sums agree bit for bit."""
import numpy as np
import pytest
import torch

from tests.conftest import has_gpu

pytestmark = pytest.mark.gpu

if has_gpu():
    import oracle
    from megatron_tensor_transformer_plan_b200 import synth, tpl
    from tests.gpu_util import assert_close_rel, make_layer, oracle_decode, to_np
    from tests.test_gpu_parity import _check_layer

    ROPE = tpl.TPL_NORM | tpl.TPL_RESIDUAL | tpl.TPL_ROPE

ONE = 0x3F80  # bf16 1.0: cache slots the call must not touch


# ---------------------------------------------------------------------------
# decode
# ---------------------------------------------------------------------------

DECODE = [
    # H, nq, nkv, F, t, B, S
    (512, 8, 2, 1376, 2, 3, 37),
    (1024, 16, 8, 2816, 8, 16, 3000),  # far position: angles of thousands of radians
    (768, 12, 4, 1056, 4, 5, 129),     # g = 3
    (256, 4, 4, 704, 4, 1, 0),         # position 0: the identity
]


@pytest.mark.parametrize("gemv_mode", [0, 3])
@pytest.mark.parametrize("case", DECODE)
def test_decode_layer_rope(gpu, case, gemv_mode):
    H, nq, nkv, F, t, B, S = case
    L = make_layer(H, nq, nkv, 128, F, t, B, S, flags=ROPE, S_cap=S + 3, seed=3)
    L.plan.set_option(tpl.TPL_OPT_GEMV_MODE, gemv_mode)
    ref_y, tr = oracle_decode(L)
    _check_layer(L, ref_y, tr)


def test_qkv_rope_without_fp32_copies(gpu):
    """Without caller k_new/v_new the rotation still starts from the unrounded
    key: cache slot S holds the bf16 rounding of the oracle's rotated key."""
    H, nq, nkv, F, t, B, S = 1024, 16, 8, 2816, 4, 4, 500
    L = make_layer(H, nq, nkv, 128, F, t, B, S, flags=ROPE, S_cap=S + 1, seed=4)
    _, tr = oracle_decode(L)
    q = torch.empty((B, nq, 128), dtype=torch.float32, device=gpu)
    L.plan.qkv(L.packed, L.kv, L.x, S, q, L.ws)
    torch.cuda.synchronize()
    from tests.gpu_util import new_kv_slot
    kk, vv = new_kv_slot(L)
    assert_close_rel(to_np(q).reshape(B, -1), tr["q"], what="q")
    assert_close_rel(to_np(kk), tr["k_new"], what="k (slot S)")
    assert_close_rel(to_np(vv), tr["v_new"], what="v (slot S)")
    # the same bits as the step with fp32 copies
    kn = torch.empty((B, nkv, 128), dtype=torch.float32, device=gpu)
    vn = torch.empty_like(kn)
    L.plan.qkv(L.packed, L.kv, L.x, S, q, L.ws, kn, vn)
    torch.cuda.synchronize()
    kk2, _ = new_kv_slot(L)
    assert torch.equal(kk, kk2) and torch.equal(kk2, kn.reshape(B, -1).bfloat16())


def test_rope_changes_the_result(gpu):
    """The flag is not a no-op: the same layer without it differs (S > 0)."""
    H, nq, nkv, F, t, B, S = 512, 8, 2, 1376, 2, 2, 40
    a = make_layer(H, nq, nkv, 128, F, t, B, S, flags=ROPE, seed=5)
    b = make_layer(H, nq, nkv, 128, F, t, B, S, seed=5)
    ya, yb = torch.empty_like(a.x), torch.empty_like(b.x)
    a.plan.decode_layer(a.packed, a.kv, a.x, S, ya, None, a.ws)
    b.plan.decode_layer(b.packed, b.kv, b.x, S, yb, None, b.ws)
    torch.cuda.synchronize()
    assert not torch.equal(ya, yb)


# ---------------------------------------------------------------------------
# prefill chunks
# ---------------------------------------------------------------------------

class Chunk:
    """One sequence (batch row 0) whose cache holds `start` earlier tokens
    (seeded N(0, 1) bf16 keys/values) and 1.0 in every later slot; a chunk of
    T new tokens."""

    def __init__(self, H, nq, nkv, F, t, T, start, *, rope=True, seed=0, attn_mode=0, pad=5, x=None):
        flags = tpl.TPL_NORM | tpl.TPL_RESIDUAL | (tpl.TPL_ROPE if rope else 0)
        self.dims = tpl.make_dims(H, nq, nkv, 128, F, 1, 1e-5, flags, rope_base=500000.0)
        self.plan = tpl.Plan(self.dims, t)
        self.plan.set_option(tpl.TPL_OPT_PREFILL_ATTN, attn_mode)
        self.t, self.T, self.start = t, T, start
        self.S_cap = start + T + pad
        self.w = synth.layer_weights(H, nq, nkv, 128, F, seed=seed, dtype=torch.bfloat16, device="cuda")
        self.packed = self.plan.pack_layer(self.w)
        self.x = synth.activations(T, H, seed=seed, layer=1, dtype=torch.bfloat16, device="cuda") if x is None else x
        kl, vl = synth.kv_cache((1, nkv, self.S_cap, 128), seed=seed, layer=7, device="cuda")
        kl.view(torch.int16)[:, :, start:] = ONE
        vl.view(torch.int16)[:, :, start:] = ONE
        self.kl, self.vl = kl, vl
        self.k, self.v = self.plan.pack_kv(kl), self.plan.pack_kv(vl)
        self.kv = tpl.Plan.kv(self.k, self.v, 1, self.S_cap)
        self.ws = self.plan.prefill_workspace(T)
        torch.cuda.synchronize()

    def run(self, mode=None, start=None):
        mode = tpl.TPL_REDUCE_FUSED if mode is None else mode
        y = torch.empty_like(self.x)
        y32 = torch.empty(self.x.shape, dtype=torch.float32, device="cuda")
        self.plan.prefill_chunk(self.packed, self.kv, self.x, self.start if start is None else start, y, y32,
                                self.ws, mode)
        torch.cuda.synchronize()
        return y, y32

    def logical_cache(self):
        d, t = self.dims, self.t
        nkv_s = d.n_kv_heads // t
        kk = self.k.view(t, 1, nkv_s, self.S_cap, 128)[:, 0].reshape(d.n_kv_heads, self.S_cap, 128)
        vv = self.v.view(t, 1, nkv_s, self.S_cap, 128)[:, 0].reshape(d.n_kv_heads, self.S_cap, 128)
        return kk, vv

    def intermediates(self):
        d, T = self.dims, self.T
        off = self.plan.prefill_intermediates(T)
        nqd = d.n_q_heads * 128

        def view(o, n, dt):
            return self.ws[o:o + n * torch.tensor([], dtype=dt).element_size()].view(dt)

        o_hi = view(off["o"], T * nqd, torch.bfloat16).view(T, nqd)
        o_lo = view(off["o_lo"], T * nqd, torch.bfloat16).view(T, nqd)
        return {"q": view(off["q"], T * nqd, torch.float32).view(T, nqd).clone(),
                "attn": (o_hi.float() + o_lo.float()).clone(),
                "h": view(off["h"], T * d.hidden, torch.float32).view(T, d.hidden).clone(),
                "act": view(off["act"], T * d.ffn, torch.bfloat16).view(T, d.ffn).clone()}

    def oracle_dims(self):
        d = self.dims
        return oracle.Dims(d.hidden, d.n_q_heads, d.n_kv_heads, d.head_dim, d.ffn, eps=float(d.rms_eps),
                           flags=int(d.flags) & (tpl.TPL_NORM | tpl.TPL_RESIDUAL | tpl.TPL_ROPE),
                           rope_base=float(d.rope_base))

    def oracle(self, rows=None):
        w = {k: synth.bits(v) for k, v in self.w.items()}
        return oracle.prefill_chunk(self.oracle_dims(), w, to_np(self.x), self.start, synth.bits(self.kl)[0],
                                    synth.bits(self.vl)[0], rows=rows, trace=True)


def check_chunk(C: Chunk, rows=None):
    kl0, vl0 = C.kl[0].clone(), C.vl[0].clone()
    y, y32 = C.run(tpl.TPL_REDUCE_FUSED)
    inter = C.intermediates()
    ref_y, ref_k, ref_v, tr = C.oracle(rows)
    sel = slice(None) if rows is None else list(rows)
    R = ref_k.shape[0]
    kk, vv = C.logical_cache()
    s0, T = C.start, C.T
    # earlier tokens untouched, slots past the chunk untouched
    assert torch.equal(kk[:, :s0], kl0[:, :s0]) and torch.equal(vv[:, :s0], vl0[:, :s0]), "prefix changed"
    assert bool((kk[:, s0 + T:].view(torch.int16) == ONE).all()), "slots past the chunk were written"
    kc = kk[:, s0:s0 + R].permute(1, 0, 2).reshape(R, -1)
    vc = vv[:, s0:s0 + R].permute(1, 0, 2).reshape(R, -1)
    assert_close_rel(to_np(kc), ref_k, what="k (cache slots start..)")
    assert_close_rel(to_np(vc), ref_v, what="v (cache slots start..)")
    assert_close_rel(to_np(inter["q"][sel]), tr["q"], what="q")
    assert_close_rel(to_np(inter["attn"][sel]), tr["attn"], what="attention output")
    assert_close_rel(to_np(inter["h"][sel]), tr["h"], what="h")
    assert_close_rel(to_np(inter["act"][sel]), tr["act"], what="act")
    assert_close_rel(to_np(y32[sel]), ref_y, what="y32")
    ys, ys32 = C.run(tpl.TPL_REDUCE_SEPARATE)
    assert torch.equal(ys32, y32) and torch.equal(ys, y), "fused and separate reductions differ"
    assert C.plan.last_device_error() == tpl.TPL_OK
    return y32


CHUNKS = [
    # H, nq, nkv, F, t, T, start, rope, attention kernel
    (1024, 16, 4, 2816, 4, 200, 77, True, 0),    # ragged tiles, start inside a 64-key tile
    (1024, 16, 8, 2816, 8, 130, 300, True, 0),   # t = 8
    (1024, 16, 4, 2816, 4, 70, 128, True, 1),    # mma.sync attention, start on a tile edge
    (768, 12, 4, 1056, 1, 33, 100, True, 0),     # g = 3: mma.sync attention
    (512, 16, 1, 512, 1, 64, 64, False, 0),      # g = 16, no rotation
    (1024, 16, 4, 2816, 4, 150, 0, True, 0),     # start 0: a whole prompt with rotation
    (512, 8, 2, 1376, 2, 5, 1000, True, 0),      # short chunk after a long prefix
]


@pytest.mark.parametrize("case", CHUNKS)
def test_prefill_chunk(gpu, case):
    H, nq, nkv, F, t, T, start, rope, am = case
    check_chunk(Chunk(H, nq, nkv, F, t, T, start, rope=rope, attn_mode=am, seed=11))


@pytest.mark.parametrize("attn_mode", [0, 1])
def test_one_token_chunk_is_a_decode_step(gpu, attn_mode):
    """A one-token chunk at position S is the decode step at S: both match the
    oracle's decode, and each other within the tolerance (different kernels)."""
    H, nq, nkv, F, t, S = 1024, 16, 4, 2816, 4, 333
    L = make_layer(H, nq, nkv, 128, F, t, 1, S, flags=ROPE, S_cap=S + 1, seed=6)
    ref_y, _ = oracle_decode(L)
    yd = torch.empty((1, H), dtype=torch.float32, device=gpu)
    L.plan.decode_layer(L.packed, L.kv, L.x, S, torch.empty_like(L.x), yd, L.ws)
    # the same cache and weights through the chunk call (slot S rewritten)
    L.plan.set_option(tpl.TPL_OPT_PREFILL_ATTN, attn_mode)
    ws = L.plan.prefill_workspace(1)
    yc = torch.empty((1, H), dtype=torch.float32, device=gpu)
    L.plan.prefill_chunk(L.packed, L.kv, L.x, S, None, yc, ws)
    torch.cuda.synchronize()
    assert_close_rel(to_np(yd), ref_y, what="decode")
    assert_close_rel(to_np(yc), ref_y, what="one-token chunk")
    assert_close_rel(to_np(yc), to_np(yd), tol=5e-3, what="chunk vs decode")


def test_two_chunks_match_the_whole_prompt(gpu):
    """Prefilling a prompt in two chunks (the second reading the first's
    cached bf16 keys) gives the oracle's single-chunk outputs."""
    H, nq, nkv, F, t, T1, T2 = 1024, 16, 4, 2816, 4, 100, 90
    x = synth.activations(T1 + T2, H, seed=12, layer=1, dtype=torch.bfloat16, device="cuda")
    C = Chunk(H, nq, nkv, F, t, T1 + T2, 0, seed=12, x=x)
    ref_y, ref_k, _, _ = C.oracle()
    # chunk 1 then chunk 2 into the same cache
    ws1, ws2 = C.plan.prefill_workspace(T1), C.plan.prefill_workspace(T2)
    y1 = torch.empty((T1, H), dtype=torch.float32, device=gpu)
    y2 = torch.empty((T2, H), dtype=torch.float32, device=gpu)
    C.plan.prefill_chunk(C.packed, C.kv, x[:T1].contiguous(), 0, None, y1, ws1)
    C.plan.prefill_chunk(C.packed, C.kv, x[T1:].contiguous(), T1, None, y2, ws2)
    torch.cuda.synchronize()
    assert_close_rel(to_np(torch.cat([y1, y2])), ref_y, what="y (two chunks)")
    kk, _ = C.logical_cache()
    assert_close_rel(to_np(kk[:, :T1 + T2].permute(1, 0, 2).reshape(T1 + T2, -1)), ref_k, what="k")
    assert C.plan.last_device_error() == tpl.TPL_OK


def test_chunk_rejects(gpu):
    C = Chunk(512, 8, 2, 1376, 2, 16, 10, seed=1, pad=0)
    y32 = torch.empty((16, 512), dtype=torch.float32, device=gpu)
    with pytest.raises(tpl.TplError) as e:
        C.plan.prefill_chunk(C.packed, C.kv, C.x, 11, None, y32, C.ws)  # start + T > seq_cap
    assert e.value.code == tpl.TPL_ENOMEM
    with pytest.raises(tpl.TplError) as e:
        C.plan.prefill_chunk(C.packed, C.kv, C.x, -1, None, y32, C.ws)
    assert e.value.code == tpl.TPL_EINVAL


@pytest.mark.slow
def test_prefill_chunk_70b_dims(gpu):
    """70B dimensions (t = 8), a 256-token chunk after 1900 cached tokens,
    with rotation; sampled rows against the oracle."""
    C = Chunk(8192, 64, 8, 28672, 8, 256, 1900, seed=13, pad=8)
    check_chunk(C, rows=[0, 1, 127, 128, 255])
