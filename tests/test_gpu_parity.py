"""GPU (CUDA, sm_100a) vs the fp64 CPU oracle on small shapes that span several
32-token tiles, a ragged last tile and a ragged channel tile; plus the method's
invariants on the GPU and the edge cases."""
import numpy as np
import pytest

import oracle
from selective_ssm_scan_mamba_b200 import inputs as I
from tests.gpu_util import RTOL_Y, assert_c12, assert_state, to_dev, to_f64

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def bd():
    from selective_ssm_scan_mamba_b200 import bdscan
    return bdscan


def make_case(seed, Bt, L, D, N, io, gated=False, with_h0=False):
    s = I.make_sequence(seed, Bt, L, D, N, io, gated=gated)
    s.update(I.make_params(seed, D, N))
    s["h0"] = I.make_state(seed + 1, Bt, D, N, scale=0.5) if with_h0 else None
    return s


def dev(s):
    return {k: (None if v is None else to_dev(v)) for k, v in s.items()}


TRAIN_CASES = [
    # (Bt, L, D, N, K, io, gated, h0, softplus)
    (2, 96, 72, 16, 16, "f32", False, False, True),
    (2, 96, 72, 16, 16, "bf16", True, True, True),
    (1, 80, 64, 16, 4, "bf16", False, True, True),
    (2, 96, 40, 16, 32, "f32", True, True, False),
    (1, 90, 64, 16, 3, "f32", False, True, True),
    (2, 85, 24, 16, 17, "bf16", False, False, True),
    (1, 64, 16, 16, 1, "f32", False, True, True),
    (2, 144, 64, 16, 48, "f32", True, True, True),
    (1, 128, 64, 16, 64, "bf16", False, True, True),
    (1, 256, 32, 16, 256, "f32", False, False, True),
    (2, 96, 24, 64, 16, "f32", False, True, True),
    (2, 96, 40, 64, 4, "bf16", True, False, True),
    (1, 128, 16, 64, 64, "bf16", False, True, True),
    (1, 96, 32, 64, 32, "f32", True, True, True),
    (1, 70, 24, 64, 7, "f32", False, True, True),
    # N = 64 with 8 states per lane (K = 4, 16): several channel tiles, the last ragged
    (3, 160, 200, 64, 16, "bf16", True, True, True),
    (2, 100, 104, 64, 4, "f32", True, True, True),
    (1, 64, 48, 64, 16, "f32", False, False, False),
    # an odd number of 16-token blocks: the lagged schedule's last tile is half a tile
    (1, 112, 40, 64, 16, "bf16", True, True, True),
    (2, 80, 48, 16, 16, "f32", False, True, True),
    # long blocks at N = 64 (8 states per lane): three spans, and a ragged last span
    (2, 96, 24, 64, 48, "f32", False, False, True),
    (1, 200, 40, 64, 100, "bf16", True, True, True),
    # long blocks whose span checkpoints do not fit in shared memory: the two-sweep path
    (1, 512, 16, 64, 512, "bf16", True, True, True),
    (1, 288, 16, 64, 288, "f32", False, True, True),
    (1, 200, 24, 16, 100, "bf16", True, True, True),
]


@pytest.mark.parametrize("Bt,L,D,N,K,io,gated,with_h0,sp", TRAIN_CASES)
def test_train_blocks_vs_oracle(bd, Bt, L, D, N, K, io, gated, with_h0, sp):
    s = make_case(L * 31 + K * 7 + D + N, Bt, L, D, N, io, gated, with_h0)
    if not sp:
        s["dt"] = I.f32_to_bf16_bits(np.abs(oracle.decode(s["dt"])).astype(np.float32) * 0.1) \
            if io == "bf16" else (np.abs(s["dt"]) * np.float32(0.1)).astype(np.float32)
    g = dev(s)
    y, bnd, hout = bd.train_blocks(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], K, z=g.get("z"),
                                   h0=g["h0"], dt_softplus=sp, want_boundary=True, want_h_out=True)
    torch.cuda.synchronize()
    o = oracle.train_blocks(s["x"], s["dt"], s["A"], s["B"], s["C"], s["Dskip"], K, z=s.get("z"),
                            h0=s["h0"], dt_softplus=sp)
    assert_c12(to_f64(y), o["y"], RTOL_Y[io], "y")
    assert_state(to_f64(bnd), o["boundary"], "boundary states")
    assert_state(to_f64(hout), o["h_out"], "final state")


PREFILL_CASES = [
    (2, 100, 72, 16, 4, "f32", True, True),
    (1, 96, 64, 16, 32, "bf16", False, False),
    (2, 150, 40, 16, 50, "bf16", True, True),
    (1, 96, 24, 64, 16, "f32", False, True),
    (2, 64, 16, 64, 64, "bf16", True, False),
]


@pytest.mark.parametrize("Bt,L,D,N,K,io,gated,with_h0", PREFILL_CASES)
def test_prefill_vs_oracle(bd, Bt, L, D, N, K, io, gated, with_h0):
    s = make_case(L * 17 + K + D + N, Bt, L, D, N, io, gated, with_h0)
    g = dev(s)
    y, hout, bnd = bd.prefill(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], K, z=g.get("z"),
                              h0=g["h0"], want_boundary=True)
    torch.cuda.synchronize()
    o = oracle.prefill(s["x"], s["dt"], s["A"], s["B"], s["C"], s["Dskip"], K, z=s.get("z"), h0=s["h0"])
    assert_c12(to_f64(y), o["y"], RTOL_Y[io], "y")
    assert_state(to_f64(bnd), o["boundary"], "boundary states")
    assert_state(to_f64(hout), o["h_out"], "final state")


STEP_CASES = [
    (1, 32, 64, 16, "bf16", False), (3, 16, 72, 16, "f32", True), (2, 5, 40, 16, "f32", False),
    (1, 48, 64, 16, "bf16", True), (2, 32, 16, 64, "bf16", False), (1, 20, 24, 64, "f32", True),
    (1, 64, 32, 64, "bf16", True), (2, 100, 24, 16, "f32", False),
    (2, 16, 200, 64, "bf16", True), (3, 4, 72, 64, "f32", False),
    # the block step of few rows at every compiled block length, partial channel tiles
    (2, 4, 40, 16, "bf16", True), (1, 16, 24, 16, "bf16", False), (1, 32, 200, 16, "bf16", True),
    # rows of 16 channels more than the SMs, of 32 channels fewer: the 32-channel width
    (1, 32, 2392, 16, "bf16", True), (1, 7, 2392, 16, "f32", False),
]


@pytest.mark.parametrize("Bt,K,D,N,io,gated", STEP_CASES)
def test_block_step_and_commit_vs_oracle(bd, Bt, K, D, N, io, gated):
    s = make_case(K * 13 + D + N, Bt, K, D, N, io, gated, with_h0=True)
    g = dev(s)
    cache = g["h0"].clone()
    before = cache.clone()
    y = bd.block_step(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], cache, z=g.get("z"))
    torch.cuda.synchronize()
    assert torch.equal(cache, before), "block_step must not write the cache"
    o_y = oracle.block_step(s["x"], s["dt"], s["A"], s["B"], s["C"], s["Dskip"], s["h0"], z=s.get("z"))
    assert_c12(to_f64(y), o_y, RTOL_Y[io], "step y")
    # commit with y: the same y, and the cache advanced
    yc = bd.commit_block(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], cache, z=g.get("z"), want_y=True)
    torch.cuda.synchronize()
    o_h, o_yc = oracle.commit_block(s["x"], s["dt"], s["A"], s["B"], s["C"], s["Dskip"], s["h0"], z=s.get("z"))
    assert torch.equal(yc, y), "commit y must equal the step y on the same inputs"
    assert_state(to_f64(cache), o_h, "committed state")
    # commit without y takes the forward-only path: same state bit for bit
    cache2 = before.clone()
    bd.commit_block(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], cache2, z=g.get("z"))
    torch.cuda.synchronize()
    assert torch.equal(cache2, cache)


def test_block_step_channel_widths_agree_bitwise(bd):
    """A block step of few rows runs 16 or 32 channels per CTA, chosen by the row
    count. Channels are independent and both widths add a token's 16 per-state
    partials in state order, so the same channels give the same bits whichever
    width runs them: 2400 channels take the 32-channel width on 148 SMs (150
    rows of 16), their first 1536 the 16-channel width (96 rows of 16)."""
    K, wide, narrow = 32, 2400, 1536
    s = make_case(977, 1, K, wide, 16, "bf16", gated=True, with_h0=True)
    g = dev(s)
    cut = lambda t: t[..., :narrow].contiguous()  # noqa: E731
    cache_w, cache_n = g["h0"].clone(), g["h0"][:, :narrow].contiguous()
    y_w = bd.block_step(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], cache_w, z=g["z"])
    y_n = bd.block_step(cut(g["x"]), cut(g["dt"]), g["A"][:narrow].contiguous(), g["B"], g["C"],
                        g["Dskip"][:narrow].contiguous(), cache_n, z=cut(g["z"]))
    torch.cuda.synchronize()
    assert torch.equal(y_w[..., :narrow], y_n)
    yc_w = bd.commit_block(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], cache_w, z=g["z"], want_y=True)
    yc_n = bd.commit_block(cut(g["x"]), cut(g["dt"]), g["A"][:narrow].contiguous(), g["B"], g["C"],
                           g["Dskip"][:narrow].contiguous(), cache_n, z=cut(g["z"]), want_y=True)
    torch.cuda.synchronize()
    assert torch.equal(yc_w[..., :narrow], yc_n)
    assert torch.equal(cache_w[:, :narrow], cache_n)


@pytest.mark.parametrize("io,N,K", [("bf16", 16, 32), ("f32", 16, 16), ("bf16", 64, 16), ("f32", 64, 4)])
def test_cache_exactness_on_gpu(bd, io, N, K):
    """Committing blocks one by one reproduces the one-shot prefill's boundary
    states bit for bit, and the training pass emits the same states."""
    Bt, L, D = 2, 8 * K, 64 if N == 16 else 32
    s = make_case(900 + K + N, Bt, L, D, N, io, gated=False, with_h0=True)
    g = dev(s)
    _, hout, bnd = bd.prefill(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], K, h0=g["h0"],
                              want_y=False, want_boundary=True)
    _, tb, th = bd.train_blocks(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], K, h0=g["h0"],
                                want_boundary=True, want_h_out=True)
    cache = g["h0"].clone()
    for j in range(L // K):
        sl = slice(j * K, (j + 1) * K)
        blk = {k: g[k][:, sl].contiguous() for k in ("x", "dt", "B", "C")}
        # a few denoising steps with other inputs must leave the cache alone
        for st in range(3):
            noisy = dev(I.make_sequence(77 + st, Bt, K, D, N, io, stream=("noisy", j, st)))
            bd.block_step(noisy["x"], noisy["dt"], g["A"], noisy["B"], noisy["C"], g["Dskip"], cache)
        bd.commit_block(blk["x"], blk["dt"], g["A"], blk["B"], blk["C"], g["Dskip"], cache)
        torch.cuda.synchronize()
        assert torch.equal(cache, bnd[:, j]), f"commit {j} differs from the prefill boundary state"
        assert torch.equal(tb[:, j], bnd[:, j])
    assert torch.equal(cache, hout) and torch.equal(th, hout)
    o = oracle.prefill(s["x"], s["dt"], s["A"], s["B"], s["C"], s["Dskip"], K, h0=s["h0"])
    assert_state(to_f64(bnd), o["boundary"], "boundary states vs oracle")


def test_block_locality_and_prefix_only_on_gpu(bd):
    Bt, L, D, N, K, io = 1, 128, 64, 16, 16, "bf16"
    s = make_case(4242, Bt, L, D, N, io)
    g = dev(s)
    y0, b0, _ = bd.train_blocks(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], K, want_boundary=True)
    j = 3
    p = {k: g[k].clone() for k in ("x", "dt", "B", "C")}
    for k in p:   # change every token after block j
        p[k][:, (j + 1) * K:] = -p[k][:, (j + 1) * K:]
    y1, b1, _ = bd.train_blocks(p["x"], p["dt"], g["A"], p["B"], p["C"], g["Dskip"], K, want_boundary=True)
    torch.cuda.synchronize()
    assert torch.equal(b1[:, : j + 1], b0[:, : j + 1]), "states up to block j depend only on the prefix"
    assert torch.equal(y1[:, : (j + 1) * K], y0[:, : (j + 1) * K]), "outputs of blocks <= j depend only on the prefix"


def test_deterministic(bd):
    s = make_case(5, 4, 256, 128, 16, "bf16", gated=True, with_h0=True)
    g = dev(s)
    outs = [bd.train_blocks(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], 16, z=g["z"], h0=g["h0"],
                            want_boundary=True, want_h_out=True) for _ in range(2)]
    torch.cuda.synchronize()
    for a, b in zip(outs[0], outs[1]):
        assert torch.equal(a, b)


def test_empty_sequence_returns_initial_state(bd):
    s = make_case(6, 2, 0, 64, 16, "f32", with_h0=True)
    g = dev(s)
    y, hout, _ = bd.prefill(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], 16, h0=g["h0"])
    torch.cuda.synchronize()
    assert y.numel() == 0 and torch.equal(hout, g["h0"])
    y, _, hout = bd.train_blocks(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], 16, want_h_out=True)
    torch.cuda.synchronize()
    assert torch.count_nonzero(hout) == 0


def test_empty_batch(bd):
    s = make_case(7, 0, 32, 64, 16, "bf16")
    g = dev(s)
    y, _, _ = bd.train_blocks(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], 16)
    assert y.numel() == 0


def test_errors_are_raised(bd):
    s = make_case(8, 1, 64, 64, 16, "bf16")
    g = dev(s)
    with pytest.raises(bd.BdscanError, match="INVALID_ARG"):
        bd.train_blocks(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], 24)   # 64 % 24 != 0
    with pytest.raises(bd.BdscanError, match="UNSUPPORTED"):
        bd.train_blocks(g["x"][:, :0].contiguous(), g["dt"][:, :0].contiguous(), g["A"], g["B"][:, :0].contiguous(),
                        g["C"][:, :0].contiguous(), g["Dskip"], 4096)   # block too long for the long path
    s2 = make_case(9, 1, 32, 64, 16, "f32")
    g2 = dev(s2)
    A32 = torch.zeros(64, 32, device="cuda")
    B32 = torch.zeros(1, 32, 32, device="cuda")
    with pytest.raises(bd.BdscanError, match="UNSUPPORTED"):
        bd.train_blocks(g2["x"], g2["dt"], A32, B32, B32, g2["Dskip"], 16)
    with pytest.raises(ValueError):
        bd.train_blocks(g2["x"][:, ::2], g2["dt"], g2["A"], g2["B"], g2["C"], g2["Dskip"], 16)


@pytest.mark.parametrize("Bt,L,D,N,K,io,gated,with_h0", [
    (1, 4096, 64, 16, 32, "bf16", False, True), (2, 3000, 40, 16, 8, "f32", True, False),
    (1, 2048, 32, 64, 16, "bf16", True, True), (1, 520, 64, 16, 4, "f32", False, True),
])
def test_prefill_chunked_vs_oracle_and_sequential(bd, Bt, L, D, N, K, io, gated, with_h0):
    s = make_case(L + D + K, Bt, L, D, N, io, gated, with_h0)
    g = dev(s)
    need = bd.prefill_chunked_workspace_bytes(g["x"], g["B"], K)
    assert need > 0, "these sizes should take the chunked path"
    y, hout, bnd = bd.prefill_chunked(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], K, z=g.get("z"),
                                      h0=g["h0"], want_boundary=True)
    ys, hs, bs = bd.prefill(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], K, z=g.get("z"), h0=g["h0"],
                            want_boundary=True)
    torch.cuda.synchronize()
    o = oracle.prefill(s["x"], s["dt"], s["A"], s["B"], s["C"], s["Dskip"], K, z=s.get("z"), h0=s["h0"])
    assert_c12(to_f64(y), o["y"], RTOL_Y[io], "y")
    assert_state(to_f64(bnd), o["boundary"], "boundary states")
    assert_state(to_f64(hout), o["h_out"], "final state")
    assert_state(to_f64(bnd), to_f64(bs), "chunked vs sequential states")


def test_prefill_chunked_single_chunk_is_sequential(bd):
    s = make_case(77, 8, 256, 1536, 16, "bf16", with_h0=True)
    g = dev(s)
    assert bd.prefill_chunked_workspace_bytes(g["x"], g["B"], 16) == 0
    y, h, b = bd.prefill_chunked(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], 16, h0=g["h0"], want_boundary=True)
    ys, hs, bs = bd.prefill(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], 16, h0=g["h0"], want_boundary=True)
    torch.cuda.synchronize()
    assert torch.equal(y, ys) and torch.equal(h, hs) and torch.equal(b, bs)


def test_prefill_chunked_rejects_small_workspace(bd):
    s = make_case(78, 1, 4096, 64, 16, "bf16")
    g = dev(s)
    need = bd.prefill_chunked_workspace_bytes(g["x"], g["B"], 16)
    with pytest.raises(bd.BdscanError, match="WORKSPACE"):
        bd.prefill_chunked(g["x"], g["dt"], g["A"], g["B"], g["C"], g["Dskip"], 16,
                           ws=torch.empty(need - 16, dtype=torch.uint8, device="cuda"))
