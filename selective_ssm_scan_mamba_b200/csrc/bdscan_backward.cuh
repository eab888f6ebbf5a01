// Backward pass of the all-block training scan (sm_100a).
//
// The forward pass (abstract and "Methodik" of "Training Hybrid Block
// Diffusion Language Models with Partial Bidirectionality"): per channel d and
// state n,
//     h_t = a_t h_{t-1} + b_t                      over the whole sequence
//     g_t = a_t g_{t+1} + b_t, zero after each block end
//     s_t = sum_n C_t (h_t + g_t) + 2 Dskip x_t,   y_t = s_t * gate_t
// with a_t = exp(delta_t A), b_t = delta_t x_t B_t. Its adjoint, given dy:
//     ds_t     = dy_t gate_t
//     lambda_t = ds_t C_t + a_{t+1} lambda_{t+1}   (dL/dh_t, whole sequence)
//     mu_t     = ds_t C_t + a_{t-1} mu_{t-1}       (dL/dg_t, inside the block)
//     db_t = lambda_t + mu_t,  da_t = lambda_t h_{t-1} + mu_t g_{t+1}
// and from them dx, d(dt), dz, dB, dC, dA, dDskip and dh0 = a_0 lambda_0.
//
// Work decomposition
//   grid   = (ceil(D / 32), batch); lane = channel, warp = 4 states, as in the
//            forward kernel. A CTA walks its sequence from the end backwards.
//   tiles  = 8 tokens. A segment starts at a block start: whole blocks up to
//            8 tokens (K <= 8) or one block (K > 8). The forward state at a
//            segment start is the forward pass's block-boundary state (h0 for
//            the first), so no forward state is stored by the forward pass
//            beyond the caches it writes anyway. At N = 16 that state is copied
//            into the ring stage of the segment's first tile with the tile's
//            inputs (cp.async, two steps ahead), so no tile waits on a global
//            load of it; at N = 64 the dB | dC tile leaves no room and it is
//            loaded directly.
//   long   = for K > 8 the block's tiles are first swept forwards (phase 1) to
//            leave (h, a_t mu_t) checkpoints at tile starts in the workspace;
//            the tiles then run last to first (phase 2).
//   phase 2= per tile: a forward sweep recomputes a_t, b_t, h_{t-1} and mu_t
//            and keeps them in Tensor Memory (16 columns per token); a backward
//            sweep then runs the two adjoint chains (g and lambda), forms the
//            per-state gradient terms and reduces them:
//            * over states (dx, d delta, the pre-gate sum s for dz): per-warp
//              partials through a padded shared-memory buffer, as the forward
//              readout does;
//            * over channels (dB, dC, which B and C share across D): each
//              lane's per-state terms go to a padded shared-memory tile that
//              is summed over the CTA's 32 channels into one partial row per
//              token in the workspace; bdscan_bwd_reduce sums the CTAs' rows
//              in a fixed order (no float atomics, so the result is bitwise
//              deterministic).
//   block starts / ends inside a tile are bit masks formed once per tile;
//   every per-token update runs on packed fp32x2 (two states per instruction).
//   dA, dDskip = per-(batch row, channel) partials in the workspace, summed
//            over the batch by bdscan_bwd_reduce.
#pragma once

#include "bdscan_kernels.cuh"

namespace bdk {

struct BwdArgs {
    const void *x, *dt, *B, *C, *z, *dy;
    const float *A, *Dskip, *h0, *boundary;
    void *dx, *ddt, *dz;
    float *dh0;
    float *ws_bc;   // [batch, ctiles, L, 2N]  per-CTA partial dB | dC rows
    float *ws_a;    // [batch, D, N]           per-row partial dA
    float *ws_d;    // [batch, D]              per-row partial dDskip
    float *ws_ck;   // [batch, ctiles, nck, W, 32, 8]  tile checkpoints inside long blocks
    int64_t L, D, nck;
    int32_t K, dt_softplus;
};

template <int N>
struct BwdCfg {
    static constexpr int NPT = 4;
    static constexpr int W = N / NPT;                  // warps (state groups)
    static constexpr int THREADS = 32 * W;
    static constexpr int TT = 8;                       // tokens per tile
    static constexpr int S = 3;                        // cp.async ring depth
    static constexpr int BR = 2 * N + 4;               // padded per-lane row of the dB | dC tile
    static constexpr int WCOLS = TT * 16;              // TMEM columns per warp: a, b, h_prev, mu per token
    static constexpr int TNEED = ((W + 3) / 4) * WCOLS;
    static constexpr int TCOLS = TNEED <= 32 ? 32 : (TNEED <= 64 ? 64 : (TNEED <= 128 ? 128 : (TNEED <= 256 ? 256 : 512)));
    static constexpr int MINB = THREADS >= 512 ? 1 : 3;
    static constexpr int PER = TT / W > 0 ? TT / W : 1;   // readout tokens per warp
    static_assert(TNEED <= 512, "TMEM columns");
};

template <class IO, int N>
struct BwdLayout {
    using CF = BwdCfg<N>;
    static constexpr int TT = CF::TT, W = CF::W;
    static constexpr int xb = TT * kCh * (int)sizeof(IO);   // one x / dt / z / dy tile
    static constexpr int bb = TT * N * (int)sizeof(IO);     // one B / C tile
    // the segment's start state [W][32][4], staged with a segment's first tile
    // (N = 16 only: at N = 64 the dB | dC tile leaves no room for it)
    static constexpr bool HS = N == 16;
    static constexpr int hs = 4 * xb + 2 * bb;
    static constexpr int stage = hs + (HS ? W * kCh * 16 : 0);
    static constexpr int dq = CF::S * stage;                // float4 (delta, delta*x, ds, d delta/d dt) [TT][32]
    static constexpr int bf = dq + TT * kCh * 16;           // float B  [TT][N]
    static constexpr int cf = bf + TT * N * 4;              // float C  [TT][N]
    static constexpr int red = cf + TT * N * 4;             // float [3][W][TT][32]: P, Q, S partials
    static constexpr int bc = red + 3 * W * TT * kCh * 4;   // float [TT][32][BR]: per-lane dB | dC terms
    static constexpr int dsk = bc + TT * kCh * CF::BR * 4;  // float [W][32]: dDskip partials
    static constexpr int bytes = dsk + W * kCh * 4;
    static_assert(xb % 16 == 0 && bb % 16 == 0 && (CF::BR * 4) % 16 == 0, "16-byte rows");
};

// Copy tokens [t0, t0 + tlen) of x, dt, z, dy, B, C into a ring stage
// (rows past tlen and channels past D zero-filled without a global read).
template <class IO, int N, int TT, int NT>
__device__ __forceinline__ void stage_bwd_tile(char *st, const BwdArgs &a, int64_t b, int64_t d0, int64_t t0,
                                               int tlen, bool gated) {
    constexpr int EPC = 16 / (int)sizeof(IO);
    constexpr int XC = kCh / EPC;
    constexpr int BC = N / EPC;
    IO *xs = reinterpret_cast<IO *>(st);
    IO *dts = xs + TT * kCh;
    IO *zs = dts + TT * kCh;
    IO *dys = zs + TT * kCh;
    IO *Bs = dys + TT * kCh;
    IO *Cs = Bs + TT * N;
    const int64_t row0 = b * a.L + t0;
    for (int e = threadIdx.x; e < TT * XC; e += NT) {
        const int t = e / XC, ch = e % XC;
        const int64_t d = d0 + (int64_t)ch * EPC;
        const bool ok = t < tlen && d < a.D;
        const int64_t off = ok ? ((row0 + t) * a.D + d) : 0;
        const int so = t * kCh + ch * EPC;
        cp_async16(xs + so, static_cast<const IO *>(a.x) + off, ok);
        cp_async16(dts + so, static_cast<const IO *>(a.dt) + off, ok);
        cp_async16(dys + so, static_cast<const IO *>(a.dy) + off, ok);
        if (gated) cp_async16(zs + so, static_cast<const IO *>(a.z) + off, ok);
    }
    for (int e = threadIdx.x; e < TT * BC; e += NT) {
        const int t = e / BC, ch = e % BC;
        const bool ok = t < tlen;
        const int64_t off = ok ? ((row0 + t) * N + (int64_t)ch * EPC) : 0;
        const int so = t * N + ch * EPC;
        cp_async16(Bs + so, static_cast<const IO *>(a.B) + off, ok);
        cp_async16(Cs + so, static_cast<const IO *>(a.C) + off, ok);
    }
}

// sigmoid(v) = 1 / (1 + 2^(-v log2 e)) on the special-function unit
__device__ __forceinline__ float sigmoid_f32(float v) {
    return rcp_approx(__fadd_rn(1.f, ex2_approx(__fmul_rn(-v, kLog2e))));
}

__device__ __forceinline__ float2 f2(float v) { return make_float2(v, v); }

// Schedule of one CTA: segments from last to first; a segment of a long block
// (K > TT) is (ntb - 1) forward tiles (phase 1) then its ntb tiles from last
// to first (phase 2); a short-block segment is one tile of whole blocks.
struct BwdTile {
    int64_t t0, ts;   // first token of the tile, of its segment
    int tlen, i, tmod;   // tokens, tile index in the segment, offset of t0 inside its block
    bool ph1;
};

__device__ __forceinline__ BwdTile bwd_tile(int q, int r, int ntb, int64_t SL, int64_t L, bool longb, int TT) {
    BwdTile t;
    t.ph1 = r < ntb - 1;
    t.i = t.ph1 ? r : 2 * ntb - 2 - r;
    t.ts = (int64_t)q * SL;
    t.t0 = t.ts + (int64_t)t.i * TT;
    const int64_t send = t.ts + SL < L ? t.ts + SL : L;
    const int64_t rem = send - t.t0;
    t.tlen = (int)(rem < TT ? rem : TT);
    t.tmod = longb ? t.i * TT : 0;
    return t;
}

template <class IO, int N>
__global__ void __launch_bounds__(BwdCfg<N>::THREADS, BwdCfg<N>::MINB) bdscan_bwd_kernel(const BwdArgs a) {
    using CF = BwdCfg<N>;
    using LY = BwdLayout<IO, N>;
    constexpr int NPT = CF::NPT, W = CF::W, NT = CF::THREADS, TT = CF::TT, S = CF::S, BR = CF::BR, PER = CF::PER;
    static_assert(NPT == 4, "two packed pairs per lane");

    extern __shared__ __align__(16) char smem[];
    float4 *dq = reinterpret_cast<float4 *>(smem + LY::dq);
    float *Bf = reinterpret_cast<float *>(smem + LY::bf);
    float *Cf = reinterpret_cast<float *>(smem + LY::cf);
    float *red = reinterpret_cast<float *>(smem + LY::red);
    float *bcr = reinterpret_cast<float *>(smem + LY::bc);
    float *dsk = reinterpret_cast<float *>(smem + LY::dsk);

    const int tid = threadIdx.x, c = tid & 31, warp = tid >> 5;
    const int n0 = warp * NPT;
    const int64_t b = blockIdx.y, ct = blockIdx.x, CT = gridDim.x;
    const int64_t d0 = ct * kCh, d = d0 + c;
    const bool dvalid = d < a.D;
    const int64_t L = a.L;
    const int K = a.K;
    const bool gated = a.z != nullptr;
    const float dskip = dvalid ? a.Dskip[d] : 0.f;
    const float dfac = __fmul_rn(2.f, dskip);

    float al[NPT];
    float2 Av2[2], rho2[2], g2[2], dA2[2], h2[2], nu2[2];
#pragma unroll
    for (int p = 0; p < 2; ++p) {
        Av2[p] = dvalid ? make_float2(a.A[d * N + n0 + 2 * p], a.A[d * N + n0 + 2 * p + 1]) : f2(0.f);
        al[2 * p] = __fmul_rn(Av2[p].x, kLog2e);
        al[2 * p + 1] = __fmul_rn(Av2[p].y, kLog2e);
        rho2[p] = f2(0.f);   // a_{t+1} lambda_{t+1}: the forward-state adjoint carried to token t
        g2[p] = f2(0.f);     // g_{t+1}
        dA2[p] = f2(0.f);
        h2[p] = f2(0.f);
        nu2[p] = f2(0.f);    // a_{t-1} mu_{t-1}: the reverse-state adjoint carried to token t
    }
    float dskacc = 0.f;

    __shared__ uint32_t tmem_slot;
    if (warp == 0) tmem_alloc(&tmem_slot, CF::TCOLS);
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tw = tmem_slot + ((uint32_t)((warp % 4) * 32) << 16) + (uint32_t)((warp / 4) * CF::WCOLS);

    const bool longb = K > TT;
    const int64_t SL = longb ? (int64_t)K : (int64_t)(TT / K) * K;   // segment length, a multiple of K
    const int nseg = (int)((L + SL - 1) / SL);
    const int ntb = longb ? (K + TT - 1) / TT : 1;                    // tiles per segment
    const int spseg = 2 * ntb - 1;
    const int64_t nblk = L / K;
    // current step (q, r) and the prefetch pointer (iq, ir), S - 1 steps ahead
    int q = nseg - 1, r = 0, iq = nseg - 1, ir = 0;
    auto advance = [&](int &qq, int &rr) {
        if (++rr == spseg) { rr = 0; --qq; }
    };
    auto issue = [&](int slot) {
        if (iq >= 0) {
            const BwdTile tl = bwd_tile(iq, ir, ntb, SL, L, longb, TT);
            stage_bwd_tile<IO, N, TT, NT>(smem + slot * LY::stage, a, b, d0, tl.t0, tl.tlen, gated);
            if (LY::HS && tl.i == 0) {   // the forward state at the segment start, staged with its first tile
                const float *src = tl.ts == 0 ? (a.h0 ? a.h0 + (b * a.D + d) * N + n0 : nullptr)
                                              : a.boundary + ((b * nblk + tl.ts / K - 1) * a.D + d) * N + n0;
                const bool ok = dvalid && src != nullptr;
                cp_async16(smem + slot * LY::stage + LY::hs + tid * 16, ok ? static_cast<const void *>(src) : a.x, ok);
            }
            advance(iq, ir);
        }
        cp_async_commit();
    };
    float *ck_base = a.ws_ck ? a.ws_ck + (((b * CT + ct) * a.nck * W + warp) * kCh + c) * 8 : nullptr;
    const int64_t ck_stride = (int64_t)W * kCh * 8;   // between consecutive checkpoints of this lane
    auto init_segment = [&](const char *st, int64_t ts) {   // forward state at a block start, reverse adjoint zero
        if constexpr (LY::HS) {
            const float4 hv = *reinterpret_cast<const float4 *>(st + LY::hs + tid * 16);
            h2[0] = make_float2(hv.x, hv.y);
            h2[1] = make_float2(hv.z, hv.w);
        } else {
            const float *src = ts == 0 ? (a.h0 ? a.h0 + (b * a.D + d) * N + n0 : nullptr)
                                       : a.boundary + ((b * nblk + ts / K - 1) * a.D + d) * N + n0;
#pragma unroll
            for (int p = 0; p < 2; ++p) h2[p] = (dvalid && src) ? make_float2(src[2 * p], src[2 * p + 1]) : f2(0.f);
        }
        nu2[0] = f2(0.f);
        nu2[1] = f2(0.f);
    };

    const float4 *dqc = dq + c;
    const float *Bw = Bf + n0;
    const float *Cw = Cf + n0;

#pragma unroll 1
    for (int s = 0; s < S - 1; ++s) issue(s);

#pragma unroll 1
    for (int s = 0; q >= 0; ++s, advance(q, r)) {
        const BwdTile tl = bwd_tile(q, r, ntb, SL, L, longb, TT);
        const int tlen = tl.tlen;
        cp_async_wait<S - 2>();
        __syncthreads();
        issue((s + S - 1) % S);
        const char *st = smem + (s % S) * LY::stage;
        const IO *xs = reinterpret_cast<const IO *>(st);
        const IO *dts = xs + TT * kCh;
        const IO *zs = dts + TT * kCh;
        const IO *dys = zs + TT * kCh;

        // block starts / ends inside the tile (bit e = token e)
        uint32_t smask = 0, emask = 0;
        if (longb) {
            if (tl.tmod == 0) smask = 1u;
            const int ee = K - 1 - tl.tmod;
            if (ee < tlen) emask = 1u << ee;
        } else {
            for (int e = 0; e < tlen; e += K) {
                smask |= 1u << e;
                emask |= 1u << (e + K - 1);
            }
        }

        // ---- per-element preprocessing: delta, delta*x, ds = dy * gate ----------
        {
            const IO *Bs = dys + TT * kCh;
            const IO *Cs = Bs + TT * N;
            for (int e = tid; e < TT * kCh; e += NT) {
                const float xv = to_f32(xs[e]);
                const float dr = to_f32(dts[e]);
                float sg = 1.f;   // d delta / d dt
                const float dl = a.dt_softplus ? softplus_sigmoid_f32(dr, sg) : dr;
                const float dyv = to_f32(dys[e]);
                const float dsv = gated ? __fmul_rn(dyv, silu_f32(to_f32(zs[e]))) : dyv;
                dq[e] = make_float4(dl, __fmul_rn(dl, xv), dsv, sg);
            }
            constexpr int EPC = 16 / (int)sizeof(IO);
            for (int e = tid; e < TT * N / EPC; e += NT) {
                widen16(Bs + e * EPC, Bf + e * EPC);
                widen16(Cs + e * EPC, Cf + e * EPC);
            }
        }
        __syncthreads();

        // ---- state at the tile start -------------------------------------------
        if (tl.i == 0) {
            init_segment(st, tl.ts);
        } else if (!tl.ph1 && tl.i < ntb - 1) {   // (tile ntb-1 continues from phase 1's registers)
            const float4 hv = *reinterpret_cast<const float4 *>(ck_base + (tl.i - 1) * ck_stride);
            const float4 nv = *reinterpret_cast<const float4 *>(ck_base + (tl.i - 1) * ck_stride + 4);
            h2[0] = make_float2(hv.x, hv.y);
            h2[1] = make_float2(hv.z, hv.w);
            nu2[0] = make_float2(nv.x, nv.y);
            nu2[1] = make_float2(nv.z, nv.w);
        }

        // A tile of a long-block segment is full whenever the block length is a
        // multiple of the tile, and holds at most the block's first token (at 0)
        // and its last (at tlen - 1): those tiles run both sweeps without
        // per-token guards, the block-start and block-end resets hoisted.
        const bool fast = longb && tlen == TT;

        // ---- forward sweep over the tile (phase 1: state only; phase 2: into TMEM)
        auto fwd_sweep = [&](auto fast_tag, auto store_tag) {
            constexpr bool FAST = decltype(fast_tag)::value, STORE = decltype(store_tag)::value;
            if (FAST && (smask & 1u)) {
                nu2[0] = f2(0.f);
                nu2[1] = f2(0.f);
            }
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            if (FAST || t < tlen) {
                const float4 q4 = dqc[t * kCh];
                const float4 Cv = *reinterpret_cast<const float4 *>(Cw + t * N);
                float at[NPT], bq[NPT];
                decay_input<NPT>(al, make_float2(q4.x, q4.y), Bw + t * N, at, bq);
                if (!FAST && ((smask >> t) & 1u)) {
                    nu2[0] = f2(0.f);
                    nu2[1] = f2(0.f);
                }
                const float2 ds2 = f2(q4.z);
                const float2 C2[2] = {make_float2(Cv.x, Cv.y), make_float2(Cv.z, Cv.w)};
                float va[8], vh[8];
#pragma unroll
                for (int p = 0; p < 2; ++p) {
                    const float2 a2 = make_float2(at[2 * p], at[2 * p + 1]);
                    const float2 b2 = make_float2(bq[2 * p], bq[2 * p + 1]);
                    const float2 mu2 = __ffma2_rn(ds2, C2[p], nu2[p]);
                    va[2 * p] = a2.x; va[2 * p + 1] = a2.y;
                    va[4 + 2 * p] = b2.x; va[5 + 2 * p] = b2.y;
                    vh[2 * p] = h2[p].x; vh[2 * p + 1] = h2[p].y;
                    vh[4 + 2 * p] = mu2.x; vh[5 + 2 * p] = mu2.y;
                    nu2[p] = __fmul2_rn(a2, mu2);
                    h2[p] = __ffma2_rn(a2, h2[p], b2);
                }
                if (STORE) {
                    tmem_st8(tw + t * 16, va);
                    tmem_st8(tw + t * 16 + 8, vh);
                }
            }
        }
        };
        if (tl.ph1) {
            if (fast) fwd_sweep(std::true_type{}, std::false_type{});
            else fwd_sweep(std::false_type{}, std::false_type{});
        } else {
            if (fast) fwd_sweep(std::true_type{}, std::true_type{});
            else fwd_sweep(std::false_type{}, std::true_type{});
        }
        if (tl.ph1) {
            if (tl.i + 1 < ntb - 1) {
                float *p = ck_base + tl.i * ck_stride;
                *reinterpret_cast<float4 *>(p) = make_float4(h2[0].x, h2[0].y, h2[1].x, h2[1].y);
                *reinterpret_cast<float4 *>(p + 4) = make_float4(nu2[0].x, nu2[0].y, nu2[1].x, nu2[1].y);
            }
            continue;
        }
        tmem_wait_st();

        // ---- phase 2 backward sweep: the adjoint chains --------------------------
        auto bwd_sweep = [&](auto fast_tag, auto gated_tag) {
            constexpr bool FAST = decltype(fast_tag)::value, GATED = decltype(gated_tag)::value;
            // h_t of the token being processed: the forward sweep's last state at
            // the tile end, then each token's h_{t-1} (the same packed FMA made them)
            float2 hc2[2] = {h2[0], h2[1]};
            float va[8], vh[8];
            const int tl1 = FAST ? TT - 1 : tlen - 1;
            tmem_ld8(tw + tl1 * 16, va);
            tmem_ld8(tw + tl1 * 16 + 8, vh);
            tmem_wait_ld(va, vh);
            if (FAST && ((emask >> (TT - 1)) & 1u)) {
                g2[0] = f2(0.f);
                g2[1] = f2(0.f);
            }
            float *redw = red + (warp * TT) * kCh + c;   // [q][warp][t][lane]
#pragma unroll
            for (int t = TT - 1; t >= 0; --t) {
                if (FAST || t < tlen) {
                    float na[8], nh[8];
                    if (t > 0) {   // next token's row, read while this one computes
                        tmem_ld8(tw + (t - 1) * 16, na);
                        tmem_ld8(tw + (t - 1) * 16 + 8, nh);
                    }
                    const float4 q4 = dqc[t * kCh];   // delta, delta*x, ds
                    const float4 Bv = *reinterpret_cast<const float4 *>(Bw + t * N);
                    const float4 Cv = *reinterpret_cast<const float4 *>(Cw + t * N);
                    if (!FAST && ((emask >> t) & 1u)) {
                        g2[0] = f2(0.f);
                        g2[1] = f2(0.f);
                    }
                    const float2 ds2 = f2(q4.z), dl2 = f2(q4.x), dlx2 = f2(q4.y);
                    const float2 C2[2] = {make_float2(Cv.x, Cv.y), make_float2(Cv.z, Cv.w)};
                    const float2 B2[2] = {make_float2(Bv.x, Bv.y), make_float2(Bv.z, Bv.w)};
                    float2 P2 = f2(0.f), Q2 = f2(0.f), S2 = f2(0.f), dB2[2], dC2[2];
#pragma unroll
                    for (int p = 0; p < 2; ++p) {
                        const float2 a2 = make_float2(va[2 * p], va[2 * p + 1]);
                        const float2 b2 = make_float2(va[4 + 2 * p], va[5 + 2 * p]);
                        const float2 hp2 = make_float2(vh[2 * p], vh[2 * p + 1]);
                        const float2 mu2 = make_float2(vh[4 + 2 * p], vh[5 + 2 * p]);
                        const float2 lam2 = __ffma2_rn(ds2, C2[p], rho2[p]);
                        const float2 db2 = __fadd2_rn(lam2, mu2);
                        const float2 da2 = __ffma2_rn(mu2, g2[p], __fmul2_rn(lam2, hp2));
                        const float2 gn2 = __ffma2_rn(a2, g2[p], b2);
                        const float2 hg2 = __fadd2_rn(hc2[p], gn2);
                        hc2[p] = hp2;
                        const float2 qa2 = __fmul2_rn(da2, a2);
                        P2 = __ffma2_rn(db2, B2[p], P2);
                        Q2 = __ffma2_rn(qa2, Av2[p], Q2);
                        if (GATED) S2 = __ffma2_rn(C2[p], hg2, S2);
                        dA2[p] = __ffma2_rn(qa2, dl2, dA2[p]);
                        dB2[p] = __fmul2_rn(db2, dlx2);
                        dC2[p] = __fmul2_rn(ds2, hg2);
                        rho2[p] = __fmul2_rn(a2, lam2);
                        g2[p] = gn2;
                    }
                    redw[t * kCh] = __fadd_rn(P2.x, P2.y);
                    redw[(W * TT + t) * kCh] = __fadd_rn(Q2.x, Q2.y);
                    if (GATED) redw[(2 * W * TT + t) * kCh] = __fadd_rn(S2.x, S2.y);
                    float *brow = bcr + (t * kCh + c) * BR + n0;
                    *reinterpret_cast<float4 *>(brow) = make_float4(dB2[0].x, dB2[0].y, dB2[1].x, dB2[1].y);
                    *reinterpret_cast<float4 *>(brow + N) = make_float4(dC2[0].x, dC2[0].y, dC2[1].x, dC2[1].y);
                    if (t > 0) {
                        tmem_wait_ld(na, nh);
#pragma unroll
                        for (int j = 0; j < 8; ++j) { va[j] = na[j]; vh[j] = nh[j]; }
                    }
                }
            }
        };
        if (fast) {
            if (gated) bwd_sweep(std::true_type{}, std::true_type{});
            else bwd_sweep(std::true_type{}, std::false_type{});
        } else {
            if (gated) bwd_sweep(std::false_type{}, std::true_type{});
            else bwd_sweep(std::false_type{}, std::false_type{});
        }
        __syncthreads();

        // ---- readout: dx, d(dt), dz of the tile's (token, channel) pairs ---------
        if (warp * PER < TT) {
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int t = warp * PER + i;
                if (t < tlen && dvalid) {
                    float P = 0.f, Q = 0.f, Sg = 0.f;
#pragma unroll
                    for (int gg = 0; gg < W; ++gg) {
                        const float *rr = red + (gg * TT + t) * kCh + c;
                        P = __fadd_rn(P, rr[0]);
                        Q = __fadd_rn(Q, rr[W * TT * kCh]);
                        if (gated) Sg = __fadd_rn(Sg, rr[2 * W * TT * kCh]);
                    }
                    const int e = t * kCh + c;
                    const float4 q4 = dq[e];
                    const float xv = to_f32(xs[e]);
                    const float dxv = __fmaf_rn(q4.x, P, __fmul_rn(dfac, q4.z));
                    float ddl = __fmaf_rn(xv, P, Q);
                    if (a.dt_softplus) ddl = __fmul_rn(ddl, q4.w);
                    const int64_t go = (b * L + tl.t0 + t) * a.D + d;
                    IO o;
                    from_f32(dxv, o);
                    static_cast<IO *>(a.dx)[go] = o;
                    from_f32(ddl, o);
                    static_cast<IO *>(a.ddt)[go] = o;
                    if (gated) {
                        const float zv = to_f32(zs[e]), dyv = to_f32(dys[e]);
                        const float sv = __fmaf_rn(dfac, xv, Sg);
                        const float sg = sigmoid_f32(zv);
                        const float dsilu = __fmul_rn(sg, __fmaf_rn(zv, __fsub_rn(1.f, sg), 1.f));
                        from_f32(__fmul_rn(__fmul_rn(dyv, sv), dsilu), o);
                        static_cast<IO *>(a.dz)[go] = o;
                    }
                    dskacc = __fmaf_rn(__fmul_rn(2.f, xv), q4.z, dskacc);
                }
            }
        }
        // ---- dB | dC of the tile summed over the CTA's 32 channels: one row per token
        {
            constexpr int G4 = 2 * N / 4;   // float4 groups per row
            float4 *dst = reinterpret_cast<float4 *>(a.ws_bc + ((b * CT + ct) * L + tl.t0) * 2 * N);
            for (int k = tid; k < tlen * G4; k += NT) {
                const int t = k / G4, j4 = k % G4;
                const float *src = bcr + t * kCh * BR + j4 * 4;
                const float4 v0 = *reinterpret_cast<const float4 *>(src);
                float2 lo = make_float2(v0.x, v0.y), hi = make_float2(v0.z, v0.w);
#pragma unroll 8
                for (int l = 1; l < kCh; ++l) {
                    const float4 v = *reinterpret_cast<const float4 *>(src + l * BR);
                    lo = __fadd2_rn(lo, make_float2(v.x, v.y));
                    hi = __fadd2_rn(hi, make_float2(v.z, v.w));
                }
                dst[k] = make_float4(lo.x, lo.y, hi.x, hi.y);
            }
        }
    }
    cp_async_wait<0>();
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem_slot, CF::TCOLS);

    if (dvalid) {
#pragma unroll
        for (int p = 0; p < 2; ++p) {
            if (a.dh0) {
                a.dh0[(b * a.D + d) * N + n0 + 2 * p] = rho2[p].x;
                a.dh0[(b * a.D + d) * N + n0 + 2 * p + 1] = rho2[p].y;
            }
            a.ws_a[(b * a.D + d) * N + n0 + 2 * p] = dA2[p].x;
            a.ws_a[(b * a.D + d) * N + n0 + 2 * p + 1] = dA2[p].y;
        }
    }
    dsk[warp * kCh + c] = dskacc;
    __syncthreads();
    if (warp == 0 && dvalid) {
        float v = 0.f;
#pragma unroll
        for (int gg = 0; gg < W; ++gg) v = __fadd_rn(v, dsk[gg * kCh + c]);
        a.ws_d[b * a.D + d] = v;
    }
}

// dB, dC = sum over the CTAs' partial rows; dA, dDskip = sum over the batch
// rows' partials. One thread per output, fixed summation order.
template <class IO, int N>
__global__ void __launch_bounds__(256) bdscan_bwd_reduce(const float *__restrict__ ws_bc, const float *__restrict__ ws_a,
                                                         const float *__restrict__ ws_d, void *dB, void *dC, float *dA,
                                                         float *dDskip, int64_t Bt, int64_t L, int64_t D, int64_t CT) {
    const int64_t nbc = Bt * L * 2 * N, na = D * N, total = nbc + na + D;
    for (int64_t idx = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; idx < total;
         idx += (int64_t)gridDim.x * blockDim.x) {
        if (idx < nbc) {
            const int64_t n2 = idx % (2 * N), bt = idx / (2 * N);
            const int64_t bb = bt / L, t = bt % L;
            const float *p = ws_bc + (bb * CT * L + t) * 2 * N + n2;
            float v = 0.f;
            for (int64_t q = 0; q < CT; ++q) v = __fadd_rn(v, p[q * L * 2 * N]);
            IO o;
            from_f32(v, o);
            if (n2 < N) static_cast<IO *>(dB)[bt * N + n2] = o;
            else static_cast<IO *>(dC)[bt * N + n2 - N] = o;
        } else if (idx < nbc + na) {
            const int64_t k = idx - nbc;
            float v = 0.f;
            for (int64_t q = 0; q < Bt; ++q) v = __fadd_rn(v, ws_a[q * na + k]);
            dA[k] = v;
        } else {
            const int64_t k = idx - nbc - na;
            float v = 0.f;
            for (int64_t q = 0; q < Bt; ++q) v = __fadd_rn(v, ws_d[q * D + k]);
            dDskip[k] = v;
        }
    }
}

}  // namespace bdk
