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
//            beyond the caches it writes anyway.
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
//            * over channels (dB, dC, which B and C share across D): a
//              butterfly reduce-scatter across the warp's lanes, then one
//              partial row per CTA in the workspace, summed over the CTAs by
//              bdscan_bwd_reduce in a fixed order (no float atomics, so the
//              result is bitwise deterministic).
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
    static constexpr int RP = TT + 4;                  // padded row of the readout buffer
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
    static constexpr int TT = CF::TT, W = CF::W, RP = CF::RP;
    static constexpr int xb = TT * kCh * (int)sizeof(IO);   // one x / dt / z / dy tile
    static constexpr int bb = TT * N * (int)sizeof(IO);     // one B / C tile
    static constexpr int stage = 4 * xb + 2 * bb;
    static constexpr int dq = CF::S * stage;                // float4 (delta, delta*x, ds, 0)  [TT][32]
    static constexpr int bf = dq + TT * kCh * 16;           // float B  [TT][N]
    static constexpr int cf = bf + TT * N * 4;              // float C  [TT][N]
    static constexpr int red = cf + TT * N * 4;             // float [3][W][32][RP]: P, Q, S partials
    static constexpr int bc = red + 3 * W * kCh * RP * 4;   // float [TT][2N]: the tile's dB | dC over 32 channels
    static constexpr int dsk = bc + TT * 2 * N * 4;         // float [W][32]: dDskip partials
    static constexpr int bytes = dsk + W * kCh * 4;
    static_assert(xb % 16 == 0 && bb % 16 == 0 && (RP * 4) % 16 == 0, "16-byte rows");
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

// Sum v[0..7] over the warp's 32 lanes, scattered: afterwards lane l holds
// the total of v[l >> 2] (each value in four lanes). Fixed order, so the
// result does not depend on timing.
__device__ __forceinline__ float lane_reduce_scatter8(const float (&v)[8], int lane) {
    float w4[4], w2[2];
    const bool h16 = lane & 16, h8 = lane & 8, h4 = lane & 4;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const float send = h16 ? v[k] : v[4 + k];
        const float keep = h16 ? v[4 + k] : v[k];
        w4[k] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, 16));
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
        const float send = h8 ? w4[k] : w4[2 + k];
        const float keep = h8 ? w4[2 + k] : w4[k];
        w2[k] = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, 8));
    }
    const float send = h4 ? w2[0] : w2[1];
    const float keep = h4 ? w2[1] : w2[0];
    float r = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, 4));
    r = __fadd_rn(r, __shfl_xor_sync(0xffffffffu, r, 2));
    r = __fadd_rn(r, __shfl_xor_sync(0xffffffffu, r, 1));
    return r;
}

template <class IO, int N>
__global__ void __launch_bounds__(BwdCfg<N>::THREADS, BwdCfg<N>::MINB) bdscan_bwd_kernel(const BwdArgs a) {
    using CF = BwdCfg<N>;
    using LY = BwdLayout<IO, N>;
    constexpr int NPT = CF::NPT, W = CF::W, NT = CF::THREADS, TT = CF::TT, S = CF::S, RP = CF::RP, PER = CF::PER;

    extern __shared__ __align__(16) char smem[];
    float4 *dq = reinterpret_cast<float4 *>(smem + LY::dq);
    float *Bf = reinterpret_cast<float *>(smem + LY::bf);
    float *Cf = reinterpret_cast<float *>(smem + LY::cf);
    float *red = reinterpret_cast<float *>(smem + LY::red);
    float *bcs = reinterpret_cast<float *>(smem + LY::bc);
    float *dsk = reinterpret_cast<float *>(smem + LY::dsk);

    const int tid = threadIdx.x, c = tid & 31, warp = tid >> 5;
    const int n0 = warp * NPT;
    const int64_t b = blockIdx.y, ct = blockIdx.x, CT = gridDim.x;
    const int64_t d0 = ct * kCh, d = d0 + c;
    const bool dvalid = d < a.D;
    const int64_t L = a.L, K = a.K;
    const bool gated = a.z != nullptr;
    const float dskip = dvalid ? a.Dskip[d] : 0.f;
    const float dfac = __fmul_rn(2.f, dskip);

    float Av[NPT], al[NPT], rho[NPT], g[NPT], dAacc[NPT], h[NPT], nu[NPT];
#pragma unroll
    for (int j = 0; j < NPT; ++j) {
        Av[j] = dvalid ? a.A[d * N + n0 + j] : 0.f;
        al[j] = __fmul_rn(Av[j], kLog2e);
        rho[j] = 0.f;   // a_{t+1} lambda_{t+1}: the forward-state adjoint carried to token t
        g[j] = 0.f;     // g_{t+1}
        dAacc[j] = 0.f;
        h[j] = 0.f;
        nu[j] = 0.f;    // a_{t-1} mu_{t-1}: the reverse-state adjoint carried to token t
    }
    float dskacc = 0.f;

    __shared__ uint32_t tmem_slot;
    if (warp == 0) tmem_alloc(&tmem_slot, CF::TCOLS);
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tw = tmem_slot + ((uint32_t)((warp % 4) * 32) << 16) + (uint32_t)((warp / 4) * CF::WCOLS);

    // ---- schedule: segments from last to first; a long block's segment is
    // (ntb - 1) forward tiles (phase 1) then ntb tiles last to first (phase 2)
    const bool longb = K > TT;
    const int64_t SL = longb ? K : (TT / K) * K;          // segment length, a multiple of K
    const int64_t nseg = (L + SL - 1) / SL;
    const int64_t ntb = longb ? (K + TT - 1) / TT : 1;    // tiles per segment
    const int64_t spseg = 2 * ntb - 1;
    const int64_t nsteps = nseg * spseg;
    auto tile_of = [&](int64_t s, int64_t &t0, int &tlen, bool &ph1, int64_t &i, int64_t &ts) {
        const int64_t q = nseg - 1 - s / spseg, r = s % spseg;
        ph1 = r < ntb - 1;
        i = ph1 ? r : 2 * ntb - 2 - r;
        ts = q * SL;
        t0 = ts + i * TT;
        const int64_t send = (q + 1) * SL < L ? (q + 1) * SL : L;
        const int64_t rem = send - t0;
        tlen = (int)(rem < TT ? rem : TT);
    };
    auto issue = [&](int64_t s) {
        if (s < nsteps) {
            int64_t t0, i, ts; int tlen; bool ph1;
            tile_of(s, t0, tlen, ph1, i, ts);
            stage_bwd_tile<IO, N, TT, NT>(smem + (s % S) * LY::stage, a, b, d0, t0, tlen, gated);
        }
        cp_async_commit();
    };
    const int64_t nblk = L / K;
    auto init_segment = [&](int64_t ts) {   // forward state at a block start, reverse adjoint zero
        const float *src = ts == 0 ? (a.h0 ? a.h0 + (b * a.D + d) * N + n0 : nullptr)
                                   : a.boundary + ((b * nblk + ts / K - 1) * a.D + d) * N + n0;
#pragma unroll
        for (int j = 0; j < NPT; ++j) {
            h[j] = (dvalid && src) ? src[j] : 0.f;
            nu[j] = 0.f;
        }
    };
    float *ck_base = a.ws_ck ? a.ws_ck + (((b * CT + ct) * a.nck * W + warp) * kCh + c) * 8 : nullptr;
    const int64_t ck_stride = (int64_t)W * kCh * 8;   // between consecutive checkpoints of this lane

    const float4 *dqc = dq + c;
    const float *Bw = Bf + n0;
    const float *Cw = Cf + n0;

#pragma unroll 1
    for (int s = 0; s < S - 1; ++s) issue(s);

#pragma unroll 1
    for (int64_t s = 0; s < nsteps; ++s) {
        int64_t t0, ti, ts; int tlen; bool ph1;
        tile_of(s, t0, tlen, ph1, ti, ts);
        cp_async_wait<S - 2>();
        __syncthreads();
        issue(s + S - 1);
        const char *st = smem + (s % S) * LY::stage;
        const IO *xs = reinterpret_cast<const IO *>(st);
        const IO *dts = xs + TT * kCh;
        const IO *zs = dts + TT * kCh;
        const IO *dys = zs + TT * kCh;

        // ---- per-element preprocessing: delta, delta*x, ds = dy * gate ----------
        {
            const IO *Bs = dys + TT * kCh;
            const IO *Cs = Bs + TT * N;
            for (int e = tid; e < TT * kCh; e += NT) {
                const float xv = to_f32(xs[e]);
                const float dr = to_f32(dts[e]);
                const float dl = a.dt_softplus ? softplus_f32(dr) : dr;
                const float dyv = to_f32(dys[e]);
                const float dsv = gated ? __fmul_rn(dyv, silu_f32(to_f32(zs[e]))) : dyv;
                dq[e] = make_float4(dl, __fmul_rn(dl, xv), dsv, 0.f);
            }
            constexpr int EPC = 16 / (int)sizeof(IO);
            for (int e = tid; e < TT * N / EPC; e += NT) {
                widen16(Bs + e * EPC, Bf + e * EPC);
                widen16(Cs + e * EPC, Cf + e * EPC);
            }
        }
        __syncthreads();

        // ---- state at the tile start -------------------------------------------
        if (ti == 0) {
            init_segment(ts);
        } else if (!ph1 && ti < ntb - 1) {   // (tile ntb-1 continues from phase 1's registers)
            const float4 hv = *reinterpret_cast<const float4 *>(ck_base + (ti - 1) * ck_stride);
            const float4 nv = *reinterpret_cast<const float4 *>(ck_base + (ti - 1) * ck_stride + 4);
            h[0] = hv.x; h[1] = hv.y; h[2] = hv.z; h[3] = hv.w;
            nu[0] = nv.x; nu[1] = nv.y; nu[2] = nv.z; nu[3] = nv.w;
        }

        if (ph1) {
            // ---- phase 1: forward over the tile, leaving the next tile's checkpoint
#pragma unroll
            for (int t = 0; t < TT; ++t) {
                if (t < tlen) {
                    const float4 q4 = dqc[t * kCh];
                    float at[NPT], bq[NPT];
                    decay_input<NPT>(al, make_float2(q4.x, q4.y), Bw + t * N, at, bq);
                    const bool bstart = (t0 + t) % K == 0;
#pragma unroll
                    for (int j = 0; j < NPT; ++j) {
                        const float mu = __fmaf_rn(q4.z, Cw[t * N + j], bstart ? 0.f : nu[j]);
                        nu[j] = __fmul_rn(at[j], mu);
                        h[j] = __fmaf_rn(at[j], h[j], bq[j]);
                    }
                }
            }
            if (ti + 1 < ntb - 1) {
                float *p = ck_base + ti * ck_stride;
                *reinterpret_cast<float4 *>(p) = make_float4(h[0], h[1], h[2], h[3]);
                *reinterpret_cast<float4 *>(p + 4) = make_float4(nu[0], nu[1], nu[2], nu[3]);
            }
            continue;
        }

        // ---- phase 2 (a): forward sweep, per-token a, b, h_{t-1}, mu into TMEM --
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            if (t < tlen) {
                const float4 q4 = dqc[t * kCh];
                float at[NPT], bq[NPT], va[8], vh[8];
                decay_input<NPT>(al, make_float2(q4.x, q4.y), Bw + t * N, at, bq);
                if ((t0 + t) % K == 0) {
#pragma unroll
                    for (int j = 0; j < NPT; ++j) nu[j] = 0.f;
                }
#pragma unroll
                for (int j = 0; j < NPT; ++j) {
                    const float mu = __fmaf_rn(q4.z, Cw[t * N + j], nu[j]);
                    va[j] = at[j];
                    va[4 + j] = bq[j];
                    vh[j] = h[j];
                    vh[4 + j] = mu;
                    nu[j] = __fmul_rn(at[j], mu);
                    h[j] = __fmaf_rn(at[j], h[j], bq[j]);
                }
                tmem_st8(tw + t * 16, va);
                tmem_st8(tw + t * 16 + 8, vh);
            }
        }
        tmem_wait_st();

        // ---- phase 2 (b): backward sweep, the adjoint chains --------------------
        float pq[TT], qq[TT], sq[TT];
#pragma unroll
        for (int t = TT - 1; t >= 0; --t) {
            pq[t] = 0.f;
            qq[t] = 0.f;
            sq[t] = 0.f;
            if (t < tlen) {
                float va[8], vh[8];
                tmem_ld8(tw + t * 16, va);
                tmem_ld8(tw + t * 16 + 8, vh);
                tmem_wait_ld(va, vh);
                const float4 q4 = dqc[t * kCh];   // delta, delta*x, ds
                if ((t0 + t + 1) % K == 0) {
#pragma unroll
                    for (int j = 0; j < NPT; ++j) g[j] = 0.f;
                }
                float P = 0.f, Q = 0.f, Sg = 0.f, vbc[8];
#pragma unroll
                for (int j = 0; j < NPT; ++j) {
                    const float aj = va[j], bj = va[4 + j], hp = vh[j], mu = vh[4 + j];
                    const float Cn = Cw[t * N + j], Bn = Bw[t * N + j];
                    const float lam = __fmaf_rn(q4.z, Cn, rho[j]);
                    const float db = __fadd_rn(lam, mu);
                    const float da = __fmaf_rn(mu, g[j], __fmul_rn(lam, hp));
                    const float gn = __fmaf_rn(aj, g[j], bj);
                    const float hn = __fmaf_rn(aj, hp, bj);
                    const float hg = __fadd_rn(hn, gn);
                    const float qa = __fmul_rn(da, aj);
                    P = __fmaf_rn(db, Bn, P);
                    Q = __fmaf_rn(qa, Av[j], Q);
                    Sg = __fmaf_rn(Cn, hg, Sg);
                    dAacc[j] = __fmaf_rn(qa, q4.x, dAacc[j]);
                    vbc[j] = __fmul_rn(db, q4.y);
                    vbc[4 + j] = __fmul_rn(q4.z, hg);
                    rho[j] = __fmul_rn(aj, lam);
                    g[j] = gn;
                }
                pq[t] = P;
                qq[t] = Q;
                sq[t] = Sg;
                const float r = lane_reduce_scatter8(vbc, c);
                if ((c & 3) == 0) {
                    const int k = c >> 2;
                    bcs[t * 2 * N + (k < 4 ? n0 + k : N + n0 + k - 4)] = r;
                }
            }
        }
        {
            float *r0 = red + (warp * kCh + c) * RP;
            float *r1 = r0 + W * kCh * RP;
            float *r2 = r1 + W * kCh * RP;
#pragma unroll
            for (int q = 0; q < TT / 4; ++q) {
                *reinterpret_cast<float4 *>(r0 + 4 * q) = make_float4(pq[4 * q], pq[4 * q + 1], pq[4 * q + 2], pq[4 * q + 3]);
                *reinterpret_cast<float4 *>(r1 + 4 * q) = make_float4(qq[4 * q], qq[4 * q + 1], qq[4 * q + 2], qq[4 * q + 3]);
                *reinterpret_cast<float4 *>(r2 + 4 * q) = make_float4(sq[4 * q], sq[4 * q + 1], sq[4 * q + 2], sq[4 * q + 3]);
            }
        }
        __syncthreads();

        // ---- readout: dx, d(dt), dz of the tile; dB | dC partial rows ------------
        if (warp * PER < TT) {
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int t = warp * PER + i;
                if (t < tlen && dvalid) {
                    float P = 0.f, Q = 0.f, Sg = 0.f;
#pragma unroll
                    for (int gg = 0; gg < W; ++gg) {
                        const float *rr = red + (gg * kCh + c) * RP + t;
                        P = __fadd_rn(P, rr[0]);
                        Q = __fadd_rn(Q, rr[W * kCh * RP]);
                        Sg = __fadd_rn(Sg, rr[2 * W * kCh * RP]);
                    }
                    const int e = t * kCh + c;
                    const float4 q4 = dq[e];
                    const float xv = to_f32(xs[e]);
                    const float dxv = __fmaf_rn(q4.x, P, __fmul_rn(dfac, q4.z));
                    float ddl = __fmaf_rn(xv, P, Q);
                    if (a.dt_softplus) ddl = __fmul_rn(ddl, sigmoid_f32(to_f32(dts[e])));
                    const int64_t go = (b * L + t0 + t) * a.D + d;
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
        {
            float *dst = a.ws_bc + ((b * CT + ct) * L + t0) * 2 * N;
            for (int e = tid; e < tlen * 2 * N / 4; e += NT)
                reinterpret_cast<float4 *>(dst)[e] = reinterpret_cast<const float4 *>(bcs)[e];
        }
    }
    cp_async_wait<0>();
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem_slot, CF::TCOLS);

    if (dvalid) {
#pragma unroll
        for (int j = 0; j < NPT; ++j) {
            if (a.dh0) a.dh0[(b * a.D + d) * N + n0 + j] = rho[j];
            a.ws_a[(b * a.D + d) * N + n0 + j] = dAacc[j];
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
