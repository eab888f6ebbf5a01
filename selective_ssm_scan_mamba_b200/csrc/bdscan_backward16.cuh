// Backward pass of the all-block training scan for blocks of 16 tokens at
// N = 16 (sm_100a): the adjoint of bdscan_backward.cuh, with each block staged
// and preprocessed once.
//
// The recurrences, the gradient terms and the CTA / lane / warp mapping are
// those of bdscan_bwd_kernel (adjoint of the forward pass of "Training Hybrid
// Block Diffusion Language Models with Partial Bidirectionality", abstract and
// "Methodik"): lane = channel, warp = 4 states, Tensor Memory holds a tile of 8
// tokens (a, b, h_{t-1}, mu per state: 16 columns per token), the CTA walks its
// sequence from the last block to the first.
//
// What differs is the schedule. bdscan_bwd_kernel treats a 16-token block as
// three 8-token tile steps (a forward-only sweep over the first half to reach
// the second half's start state, then each half's forward sweep into Tensor
// Memory and backward sweep), each with its own staging, preprocessing, tile
// bookkeeping and barriers. Here one ring stage holds the whole block: x, dt,
// z, dy, B, C of 16 tokens and the block's start state (the forward pass's
// boundary state, copied with the inputs). After one wait and one
// preprocessing pass the CTA runs, from shared memory:
//     forward-only sweep over tokens 0..7          (h and a*mu at token 8)
//     forward sweep over tokens 8..15 into TMEM, backward sweep 15..8
//     barrier, readout and dB | dC rows of tokens 8..15, barrier
//     forward sweep over tokens 0..7 into TMEM (from the block's start state),
//     backward sweep 7..0
//     barrier, readout and dB | dC rows of tokens 0..7
// Five barriers per block instead of nine, one schedule computation, and the
// shared-memory partial buffers (readout sums, dB | dC tile) stay 8 tokens
// long. Every half-block is full and block-aligned, so no sweep carries a
// per-token guard and the block-start / block-end resets are fixed: the
// reverse state g is zero after token 15, the reverse adjoint a*mu is zero
// before token 0. The ring has two stages (the next block is copied while this
// one is processed). The readout's P and Q partials share one float2 per
// (token, channel) (half the shared-memory loads of the readout). The
// arithmetic per token and every summation order are those of
// bdscan_bwd_kernel, so both kernels give the same bits.
#pragma once

#include "bdscan_backward.cuh"

namespace bdk {

template <class IO>
struct Bwd16Layout {
    static constexpr int N = 16, TT = 8, TB = 16, W = N / 4, S = 2;
    static constexpr int BR = 2 * N + 4;                    // padded per-lane row of the dB | dC tile
    static constexpr int xb = TB * kCh * (int)sizeof(IO);   // one x / dt / z / dy block
    static constexpr int bb = TB * N * (int)sizeof(IO);     // one B / C block
    static constexpr int hs = 4 * xb + 2 * bb;              // the block's start state [W][32][4]
    static constexpr int stage = hs + W * kCh * 16;
    static constexpr int dq = S * stage;                    // float4 (delta, delta*x, ds, d delta/d dt) [16][32]
    static constexpr int bf = dq + TB * kCh * 16;           // float B  [16][N]
    static constexpr int cf = bf + TB * N * 4;              // float C  [16][N]
    static constexpr int red = cf + TB * N * 4;             // float2 [W][8][32] (P, Q) + float [W][8][32] S partials of a half
    static constexpr int bc = red + 3 * W * TT * kCh * 4;   // float [8][32][BR]: per-lane dB | dC terms of a half
    static constexpr int dsk = bc + TT * kCh * BR * 4;      // float [W][32]: dDskip partials
    static constexpr int bytes = dsk + W * kCh * 4;
    static_assert(xb % 16 == 0 && bb % 16 == 0 && (BR * 4) % 16 == 0, "16-byte rows");
};

template <class IO>
__global__ void __launch_bounds__(128, 3) bdscan_bwd16_kernel(const BwdArgs a) {
    using LY = Bwd16Layout<IO>;
    constexpr int N = 16, NPT = 4, W = LY::W, NT = 128, TT = LY::TT, TB = LY::TB, S = LY::S, BR = LY::BR;
    constexpr int PER = TT / W;   // readout tokens per warp in a half

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
    if (warp == 0) tmem_alloc(&tmem_slot, 128);
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    const uint32_t tw = tmem_slot + ((uint32_t)(warp * 32) << 16);   // W = 4: one lane quadrant per warp

    const int64_t nblk = L / TB;
    // stage block q (its inputs and start state) into ring slot q % S
    auto issue = [&](int64_t q) {
        if (q >= 0) {
            char *st = smem + (int)(q % S) * LY::stage;
            stage_bwd_tile<IO, N, TB, NT>(st, a, b, d0, q * TB, TB, gated);
            const float *src = q == 0 ? (a.h0 ? a.h0 + (b * a.D + d) * N + n0 : nullptr)
                                      : a.boundary + ((b * nblk + q - 1) * a.D + d) * N + n0;
            const bool ok = dvalid && src != nullptr;
            cp_async16(st + LY::hs + tid * 16, ok ? static_cast<const void *>(src) : a.x, ok);
        }
        cp_async_commit();
    };

    const float4 *dqc = dq + c;
    const float *Bw = Bf + n0;
    const float *Cw = Cf + n0;
    float2 *redpq = reinterpret_cast<float2 *>(red) + (warp * TT) * kCh + c;   // [warp][t][lane]
    float *reds = red + 2 * W * TT * kCh + (warp * TT) * kCh + c;                 // [warp][t][lane]

    // forward sweep over the 8 tokens at dqc / Bw / Cw (STORE: into TMEM for the backward sweep)
    auto fwd_sweep = [&](auto store_tag) {
        constexpr bool STORE = decltype(store_tag)::value;
#pragma unroll
        for (int t = 0; t < TT; ++t) {
            const float4 q4 = dqc[t * kCh];
            const float4 Cv = *reinterpret_cast<const float4 *>(Cw + t * N);
            float at[NPT], bq[NPT];
            decay_input<NPT>(al, make_float2(q4.x, q4.y), Bw + t * N, at, bq);
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
    };

    // backward sweep over the 8 tokens held in TMEM: the adjoint chains and the
    // per-token gradient terms into the shared partial buffers
    auto bwd_sweep = [&](auto gated_tag) {
        constexpr bool GATED = decltype(gated_tag)::value;
        float2 hc2[2] = {h2[0], h2[1]};
        float va[8], vh[8];
        tmem_ld8(tw + (TT - 1) * 16, va);
        tmem_ld8(tw + (TT - 1) * 16 + 8, vh);
        tmem_wait_ld(va, vh);
#pragma unroll
        for (int t = TT - 1; t >= 0; --t) {
            float na[8], nh[8];
            if (t > 0) {   // next token's row, read while this one computes
                tmem_ld8(tw + (t - 1) * 16, na);
                tmem_ld8(tw + (t - 1) * 16 + 8, nh);
            }
            const float4 q4 = dqc[t * kCh];   // delta, delta*x, ds
            const float4 Bv = *reinterpret_cast<const float4 *>(Bw + t * N);
            const float4 Cv = *reinterpret_cast<const float4 *>(Cw + t * N);
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
            redpq[t * kCh] = make_float2(__fadd_rn(P2.x, P2.y), __fadd_rn(Q2.x, Q2.y));
            if (GATED) reds[t * kCh] = __fadd_rn(S2.x, S2.y);
            float *brow = bcr + (t * kCh + c) * BR + n0;
            *reinterpret_cast<float4 *>(brow) = make_float4(dB2[0].x, dB2[0].y, dB2[1].x, dB2[1].y);
            *reinterpret_cast<float4 *>(brow + N) = make_float4(dC2[0].x, dC2[0].y, dC2[1].x, dC2[1].y);
            if (t > 0) {
                tmem_wait_ld(na, nh);
#pragma unroll
                for (int j = 0; j < 8; ++j) { va[j] = na[j]; vh[j] = nh[j]; }
            }
        }
    };

    // dx, d(dt), dz of a half's 8 tokens (first token t0, stage rows from r0),
    // then its dB | dC terms summed over the CTA's 32 channels: one row per token
    auto finish_half = [&](const char *st, int64_t t0, int r0) {
        const IO *xs = reinterpret_cast<const IO *>(st) + r0 * kCh;
        const IO *zs = reinterpret_cast<const IO *>(st) + 2 * TB * kCh + r0 * kCh;
        const IO *dys = reinterpret_cast<const IO *>(st) + 3 * TB * kCh + r0 * kCh;
        if (dvalid) {
            const int64_t go0 = (b * L + t0 + warp * PER) * a.D + d;   // this warp's first token of the half
#pragma unroll
            for (int i = 0; i < PER; ++i) {
                const int t = warp * PER + i;
                float P = 0.f, Q = 0.f, Sg = 0.f;
#pragma unroll
                for (int gg = 0; gg < W; ++gg) {
                    const float2 pq = reinterpret_cast<const float2 *>(red)[(gg * TT + t) * kCh + c];
                    P = __fadd_rn(P, pq.x);
                    Q = __fadd_rn(Q, pq.y);
                    if (gated) Sg = __fadd_rn(Sg, red[2 * W * TT * kCh + (gg * TT + t) * kCh + c]);
                }
                const int e = t * kCh + c;
                const float4 q4 = dq[r0 * kCh + e];
                const float xv = to_f32(xs[e]);
                const float dxv = __fmaf_rn(q4.x, P, __fmul_rn(dfac, q4.z));
                float ddl = __fmaf_rn(xv, P, Q);
                if (a.dt_softplus) ddl = __fmul_rn(ddl, q4.w);
                const int64_t go = go0 + i * a.D;
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
        constexpr int G4 = 2 * N / 4;   // float4 groups per row
        float4 *dst = reinterpret_cast<float4 *>(a.ws_bc + ((b * CT + ct) * L + t0) * 2 * N);
        for (int k = tid; k < TT * G4; k += NT) {
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
    };

    issue(nblk - 1);
#pragma unroll 1
    for (int64_t q = nblk - 1; q >= 0; --q) {
        cp_async_wait<0>();
        __syncthreads();   // block q landed; block q+1 is fully done (its slot may be refilled)
        issue(q - 1);
        const char *st = smem + (int)(q % S) * LY::stage;
        const int64_t ts = q * TB;
        {   // preprocessing of the block: delta, delta*x, ds = dy * gate, d delta / d dt; B, C widened
            const IO *xs = reinterpret_cast<const IO *>(st);
            const IO *dts = xs + TB * kCh;
            const IO *zs = dts + TB * kCh;
            const IO *dys = zs + TB * kCh;
            const IO *Bs = dys + TB * kCh;
            const IO *Cs = Bs + TB * N;
            for (int e = tid; e < TB * kCh; e += NT) {
                const float xv = to_f32(xs[e]);
                const float dr = to_f32(dts[e]);
                float sg = 1.f;
                const float dl = a.dt_softplus ? softplus_sigmoid_f32(dr, sg) : dr;
                const float dyv = to_f32(dys[e]);
                const float dsv = gated ? __fmul_rn(dyv, silu_f32(to_f32(zs[e]))) : dyv;
                dq[e] = make_float4(dl, __fmul_rn(dl, xv), dsv, sg);
            }
            constexpr int EPC = 16 / (int)sizeof(IO);
            for (int e = tid; e < TB * N / EPC; e += NT) {
                widen16(Bs + e * EPC, Bf + e * EPC);
                widen16(Cs + e * EPC, Cf + e * EPC);
            }
        }
        __syncthreads();
        auto start_state = [&]() {   // the forward state at the block start; the reverse adjoint zero
            const float4 hv = *reinterpret_cast<const float4 *>(st + LY::hs + tid * 16);
            h2[0] = make_float2(hv.x, hv.y);
            h2[1] = make_float2(hv.z, hv.w);
            nu2[0] = f2(0.f);
            nu2[1] = f2(0.f);
        };
        auto half = [&](int r0) {   // point the sweeps at stage rows r0 .. r0 + 7
            dqc = dq + r0 * kCh + c;
            Bw = Bf + r0 * N + n0;
            Cw = Cf + r0 * N + n0;
        };
        // second half: reach its start state, recompute into TMEM, backward sweep
        start_state();
        half(0);
        fwd_sweep(std::false_type{});
        half(TT);
        fwd_sweep(std::true_type{});
        tmem_wait_st();
        g2[0] = f2(0.f);   // the reverse state is zero after the block's last token
        g2[1] = f2(0.f);
        if (gated) bwd_sweep(std::true_type{});
        else bwd_sweep(std::false_type{});
        __syncthreads();
        finish_half(st, ts + TT, TT);
        __syncthreads();
        // first half: from the block's start state again
        start_state();
        half(0);
        fwd_sweep(std::true_type{});
        tmem_wait_st();
        if (gated) bwd_sweep(std::true_type{});
        else bwd_sweep(std::false_type{});
        __syncthreads();
        finish_half(st, ts, 0);
    }
    cp_async_wait<0>();
    tmem_fence_before_sync();
    __syncthreads();
    tmem_fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem_slot, 128);

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

}  // namespace bdk
