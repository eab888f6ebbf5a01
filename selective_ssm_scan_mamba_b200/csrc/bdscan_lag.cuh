// The whole-block fused pass with the reverse scan one block behind the
// forward scan (sm_100a), for passes over several blocks of 16 or 32 tokens.
//
// Method: "Training Hybrid Block Diffusion Language Models with Partial
// Bidirectionality" (arXiv 2607.02805), abstract and gist.science technical
// summary ("Methodik"): a causal forward Mamba scan over the whole sequence
// plus a reverse scan confined to each block; y = y_fwd + y_rev.
//
// Why a lagged schedule. Each element-step needs one exp (special-function
// unit) for its decay and a handful of FMAs for the two chains. Computing a
// block's decays in one phase and running its two chains in the next leaves the
// SFU idle while the chains run and the FMA pipe idle while the exps run, since
// every warp of the CTA goes through the phases together. Here step i of a
// phase runs
//   * the forward chain over token i of block j: its decay and input are
//     computed now (exp on the SFU) and written to Tensor Memory, and
//   * the reverse chain over token K-1-i of block j-1: its decay and input
//     are read back from Tensor Memory, where block j-1's forward steps left
//     them,
// so every step carries both kinds of work. One block of TMEM suffices: block
// j writes token i into the slot that block j-1's token K-1-i has just been
// read from (blocks of even index use slot i for token i, blocks of odd index
// slot K-1-i). A token's output is complete once both chains have passed it:
// the forward partial of block j waits in registers for its reverse partial,
// and the sum goes straight to the shared readout buffer (one conflict-free
// scalar store per step: no register window), so the readout of a tile covers
// the window one block behind it, and a last phase runs the reverse chain of
// the final block alone. Tiles are 32 tokens for blocks of 16 and 32 (half the
// barriers per token of 16-token tiles; one CTA per SM at N = 64 idles the SM
// at every barrier). The forward chain is software-pipelined by one token: the
// decay (its exps) and input of token i+1 are formed during step i, so their
// shared-memory loads and MUFU latency overlap step i's chain work instead of
// heading the next step.
//
// Work decomposition as in bdscan_kernel: CTA = 32 channels of one sequence,
// lane = channel, warp = NPT states; tiles of T tokens (whole blocks) staged by
// 16-byte cp.async, two tiles ahead (the previous tile's stage stays for the
// lagged readout); C widened into one of two buffers by tile parity.
#pragma once

#include "bdscan_kernels.cuh"

namespace bdk {

template <int N, int KC, int NPTV>
struct LagCfg {
    static constexpr int K = KC, NPT = NPTV, W = N / NPT, THREADS = 32 * W;
    static constexpr int T = K >= 16 ? 32 : 16;                // tokens per tile (whole blocks)
    static constexpr int NBT = T / K;                            // blocks per tile
    static constexpr int S = 4;                                  // ring stages, prefetch S - 2 tiles ahead
    static constexpr int TV = 2 * NPT;                           // TMEM columns per token: a, b
    static constexpr int WCOLS = K * TV;
    static constexpr int TNEED = (W / 4) * WCOLS;
    static constexpr int TCOLS = TNEED <= 32 ? 32 : (TNEED <= 64 ? 64 : (TNEED <= 128 ? 128 : (TNEED <= 256 ? 256 : 512)));
    static constexpr int PER = T / W > 0 ? T / W : 1;            // readout tokens per warp
    static constexpr int MINB0 = THREADS >= 512 ? 1 : NPT == 8 ? 1 : (K <= 16 ? 3 : 2);
    static constexpr int MINB = 512 / TCOLS < MINB0 ? 512 / TCOLS : MINB0;
    static_assert(W % 4 == 0 && TNEED <= 512 && T % K == 0 && (NPT == 4 || NPT == 8), "lagged layout");
};

template <class IO, int N, int KC, int NPTV>
struct LagLayout {
    using CF = LagCfg<N, KC, NPTV>;
    static constexpr int T = CF::T, S = CF::S, W = CF::W;
    static constexpr int xb = T * kCh * (int)sizeof(IO);   // one x / dt / z tile
    static constexpr int bb = T * N * (int)sizeof(IO);     // one B / C tile
    static constexpr int stage = 3 * xb + 2 * bb;
    static constexpr int dd = S * stage;                   // float2 (delta, delta*x)   [T][32]
    static constexpr int bf = dd + T * kCh * 8;            // float B                  [T][N]
    static constexpr int cf = bf + T * N * 4;              // float C, two tiles       [2][T][N]
    static constexpr int red = cf + 2 * T * N * 4;         // float window partials    [W][T][32]
    static constexpr int bytes = red + W * T * kCh * 4;
    static_assert(xb % 16 == 0 && bb % 16 == 0, "16-byte rows");
};

template <class IO, int N, int KC, int NPTV>
__global__ void __launch_bounds__(LagCfg<N, KC, NPTV>::THREADS, LagCfg<N, KC, NPTV>::MINB)
    bdscan_lag_kernel(const ScanArgs a) {
    using CF = LagCfg<N, KC, NPTV>;
    using LY = LagLayout<IO, N, KC, NPTV>;
    constexpr int K = CF::K, NPT = CF::NPT, W = CF::W, NT = CF::THREADS, T = CF::T, S = CF::S;
    constexpr int NBT = CF::NBT, TV = CF::TV, PER = CF::PER;

    extern __shared__ __align__(16) char smem[];
    float2 *dd = reinterpret_cast<float2 *>(smem + LY::dd);
    float *Bf = reinterpret_cast<float *>(smem + LY::bf);
    float *Cf2 = reinterpret_cast<float *>(smem + LY::cf);
    float *red = reinterpret_cast<float *>(smem + LY::red);

    const int tid = threadIdx.x, c = tid & 31, warp = tid >> 5;
    const int n0 = warp * NPT;
    const int64_t b = blockIdx.y;
    const int64_t d0 = (int64_t)blockIdx.x * kCh;
    const int64_t d = d0 + c;
    const bool dvalid = d < a.D;
    const int64_t L = a.L;
    const bool gated = a.z != nullptr;
    const bool want_y = a.y != nullptr;
    const float dskip = dvalid ? a.Dskip[d] : 0.f;
    const float dfac = __fmul_rn(2.f, dskip);

    float al[NPT], h[NPT];
#pragma unroll
    for (int j = 0; j < NPT; ++j) {
        al[j] = dvalid ? __fmul_rn(a.A[d * N + n0 + j], kLog2e) : 0.f;
        h[j] = (dvalid && a.h0) ? a.h0[(b * a.D + d) * N + n0 + j] : 0.f;
    }

    __shared__ uint32_t tmem_slot;
    if (warp == 0) tmem_alloc(&tmem_slot, CF::TCOLS);
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tmem_w = tmem_slot + ((uint32_t)((warp % 4) * 32) << 16) + (uint32_t)((warp / 4) * CF::WCOLS);

    const int64_t nt = (L + T - 1) / T;   // tiles
    const int64_t nblk = L / K;
    auto issue = [&](int64_t s) {
        if (s < nt) {
            const int64_t t0 = s * T;
            const int tlen = (int)(L - t0 < T ? L - t0 : T);
            stage_tile<IO, N, T, NT>(smem + (s % S) * LY::stage, a, b, d0, t0, tlen, gated);
        }
        cp_async_commit();
    };
    float *bnd_ptr = (a.boundary && dvalid) ? a.boundary + (b * nblk * a.D + d) * N + n0 : nullptr;
    auto write_boundary = [&](int64_t blk) {   // forward state after the last token of block blk
        if (bnd_ptr) {
            float *p = bnd_ptr + blk * a.D * N;
#pragma unroll
            for (int q = 0; q < NPT / 4; ++q)
                *reinterpret_cast<float4 *>(p + 4 * q) = make_float4(h[4 * q], h[4 * q + 1], h[4 * q + 2], h[4 * q + 3]);
        }
    };
    auto restart_h = [&](int64_t j) {   // two-stream pass: block j starts from the clean cache at its start
        const float *src = j == 0 ? (a.h0 ? a.h0 + (b * a.D + d) * N + n0 : nullptr)
                                  : a.blk_h0 + ((b * nblk + j - 1) * a.D + d) * N + n0;
#pragma unroll
        for (int q = 0; q < NPT; ++q) h[q] = (dvalid && src) ? src[q] : 0.f;
    };
    // TMEM slot of token i of a block: slot i in blocks of even index, K-1-i in
    // blocks of odd index
    auto slot = [](bool odd, int i) -> uint32_t { return (uint32_t)(odd ? K - 1 - i : i) * TV; };

    const float2 *ddc = dd + c;
    const float *Bw = Bf + n0;

    float yfp[K];   // forward readout partials of the block whose reverse pass comes next
#pragma unroll
    for (int i = 0; i < K; ++i) yfp[i] = 0.f;
    float *redw = red + warp * T * kCh + c;   // this lane's window partials, [W][T][32]

    // One phase: the forward chain over block jf (its tokens at local offset bi * K
    // of the current tile) and the reverse chain over block jf - 1. par_tag: the
    // parity of jf when it is known at compile time (0 or 1), else -1.
    auto phase = [&](int bi, int64_t jf, int64_t cur_tile, auto f_tag, auto r_tag, auto par_tag) {
        constexpr bool F = decltype(f_tag)::value, R = decltype(r_tag)::value;
        constexpr int PAR = decltype(par_tag)::value;
        const bool fodd = PAR >= 0 ? PAR == 1 : (jf & 1) != 0;   // block jf odd (block jr = jf - 1 even)
        const int64_t jr = jf - 1;
        const float *Cc = Cf2 + (cur_tile & 1) * T * N + n0;                    // C of the current tile
        const int64_t rtile = R ? (jr * K) / T : 0;
        const float *Cr = Cf2 + (rtile & 1) * T * N + n0;                       // C of block jr's tile
        const int lr0 = R ? (int)(jr * K - rtile * T) : 0;                      // block jr's first local token
        float g[NPT];
#pragma unroll
        for (int q = 0; q < NPT; ++q) g[q] = 0.f;
        float cr[TV];
        if constexpr (R) {
            tmem_ld(tmem_w + slot(!fodd, K - 1), cr);
            tmem_wait_ld(cr);
        }
        if (F && a.blk_h0) restart_h(jf);
        float yfc[K];
        float afn[NPT], bqn[NPT];   // decay and input of the next forward token, formed a step ahead
        if constexpr (F) decay_input<NPT>(al, ddc[bi * K * kCh], Bw + bi * K * N, afn, bqn);
#pragma unroll
        for (int i = 0; i < K; ++i) {
            float nr[TV];
            if constexpr (R) {
                if (i + 1 < K) tmem_ld(tmem_w + slot(!fodd, K - 2 - i), nr);   // the next reverse token
            }
            if constexpr (F) {
                const int tl = bi * K + i;
                float af[NPT], bq[NPT], v[TV];
#pragma unroll
                for (int q = 0; q < NPT; ++q) { af[q] = afn[q]; bq[q] = bqn[q]; }
                if (i + 1 < K) decay_input<NPT>(al, ddc[(tl + 1) * kCh], Bw + (tl + 1) * N, afn, bqn);
#pragma unroll
                for (int q = 0; q < NPT; ++q) { v[q] = af[q]; v[NPT + q] = bq[q]; }
                tmem_st(tmem_w + slot(fodd, i), v);   // the slot block jr's token K-1-i was read from
                yfc[i] = scan_step<NPT>(h, af, bq, Cc + tl * N);
            }
            if constexpr (R) {
                const int ir = K - 1 - i;
                float ar[NPT], br[NPT];
#pragma unroll
                for (int q = 0; q < NPT; ++q) { ar[q] = cr[q]; br[q] = cr[NPT + q]; }
                redw[(bi * K + ir) * kCh] = __fadd_rn(yfp[ir], scan_step<NPT>(g, ar, br, Cr + (lr0 + ir) * N));
                if (i + 1 < K) {
                    tmem_wait_ld(nr);
#pragma unroll
                    for (int q = 0; q < TV; ++q) cr[q] = nr[q];
                }
            }
        }
        if constexpr (F) {
            write_boundary(jf);
            tmem_wait_st();   // the next phase's reverse chain reads these slots
#pragma unroll
            for (int i = 0; i < K; ++i) yfp[i] = yfc[i];
        }
    };

    // Readout of nwin window tokens starting at absolute token wt0 (tokens
    // before 0 skipped): the W state-group partials of every (token, channel),
    // the skip term, the gate, the store. Warp w finishes window tokens
    // [w PER, (w+1) PER): wt0 and nwin are multiples of K, and K and T of PER,
    // so a warp's tokens lie in one tile and are all in the window or all out.
    static_assert(K % PER == 0 && T % PER == 0, "a warp's readout tokens share a tile");
    auto readout = [&](int64_t wt0, int nwin) {
        __syncthreads();   // every warp's window partials are in [W][T][32]
        float ysum[PER];
#pragma unroll
        for (int i = 0; i < PER; ++i) ysum[i] = 0.f;
#pragma unroll
        for (int gg = 0; gg < W; ++gg) {
#pragma unroll
            for (int i = 0; i < PER; ++i) ysum[i] = __fadd_rn(ysum[i], red[(gg * T + warp * PER + i) * kCh + c]);
        }
        const int tw0 = warp * PER;
        const int64_t ta0 = wt0 + tw0;
        if (want_y && dvalid && tw0 < nwin && ta0 >= 0) {
            const int64_t tile = ta0 / T;   // the tokens' staging stage is still in the ring
            const int lt0 = (int)(ta0 - tile * T);
            const IO *xs = reinterpret_cast<const IO *>(smem + (int)(tile % S) * LY::stage) + lt0 * kCh + c;
            const IO *zs = xs + 2 * T * kCh;
            IO *yo = static_cast<IO *>(a.y) + (b * L + ta0) * a.D + d;
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                float v = __fmaf_rn(dfac, to_f32(xs[i * kCh]), ysum[i]);
                if (gated) v = __fmul_rn(v, silu_f32(to_f32(zs[i * kCh])));
                IO o;
                from_f32(v, o);
                yo[i * a.D] = o;
            }
        }
    };

#pragma unroll 1
    for (int s = 0; s < S - 2; ++s) issue(s);

#pragma unroll 1
    for (int64_t s = 0; s < nt; ++s) {
        const int64_t t0 = s * T;
        const int tlen = (int)(L - t0 < T ? L - t0 : T);
        cp_async_wait<S - 3>();
        __syncthreads();   // stage s landed for every thread; tile s-1 is fully done
        issue(s + S - 2);  // into the stage of tile s-2 (tile s-1's stays for its lagged readout)
        {
            const char *st = smem + (s % S) * LY::stage;
            const IO *xs = reinterpret_cast<const IO *>(st);
            const IO *dts = xs + T * kCh;
            const IO *Bs = dts + 2 * T * kCh;
            const IO *Cs = Bs + T * N;
            float *Cc = Cf2 + (s & 1) * T * N;
#pragma unroll
            for (int e = tid; e < T * kCh; e += NT) {
                const float xv = to_f32(xs[e]);
                const float dr = to_f32(dts[e]);
                const float dl = a.dt_softplus ? softplus_f32(dr) : dr;
                dd[e] = make_float2(dl, __fmul_rn(dl, xv));
            }
            constexpr int EPC = 16 / (int)sizeof(IO);
#pragma unroll
            for (int e = tid; e < T * N / EPC; e += NT) {
                widen16(Bs + e * EPC, Bf + e * EPC);
                widen16(Cs + e * EPC, Cc + e * EPC);
            }
        }
        __syncthreads();
        const int nb = tlen / K;   // blocks of this tile
        const int64_t b0 = s * NBT;
        using PEven = std::integral_constant<int, 0>;
        using POdd = std::integral_constant<int, 1>;
        using PRun = std::integral_constant<int, -1>;
        if constexpr (NBT == 2) {   // b0 is even: block b0 + bi has the parity of bi
            if (nb > 0) {
                if (s == 0) phase(0, b0, s, std::true_type{}, std::false_type{}, PEven{});
                else phase(0, b0, s, std::true_type{}, std::true_type{}, PEven{});
            }
            if (nb > 1) phase(1, b0 + 1, s, std::true_type{}, std::true_type{}, POdd{});
        } else {
#pragma unroll
            for (int bi = 0; bi < NBT; ++bi) {
                if (bi < nb) {
                    if (bi == 0 && s == 0) phase(bi, b0 + bi, s, std::true_type{}, std::false_type{}, PRun{});
                    else phase(bi, b0 + bi, s, std::true_type{}, std::true_type{}, PRun{});
                }
            }
        }
        readout((b0 - 1) * K, nb * K);
    }
    if (nblk > 0) {   // the reverse chain of the last block, then its readout
        __syncthreads();   // every warp is past the last tile's readout of the shared partials
        phase(0, nblk, nt, std::false_type{}, std::true_type{}, std::integral_constant<int, -1>{});
        readout((nblk - 1) * K, K);
    }
    cp_async_wait<0>();
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem_slot, CF::TCOLS);
    if (a.h_out && dvalid) {
        float *p = a.h_out + (b * a.D + d) * N + n0;
#pragma unroll
        for (int j = 0; j < NPT; ++j) p[j] = h[j];
    }
}

}  // namespace bdk
