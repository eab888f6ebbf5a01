// One denoising block step of few (batch, 32-channel) rows, N = 16 (sm_100a).
//
// Method: "Training Hybrid Block Diffusion Language Models with Partial
// Bidirectionality" (arXiv 2607.02805), abstract and gist.science technical
// summary ("Methodik"): a block step resumes the causal forward scan from the
// cached forward-only state of the clean prefix and runs the reverse scan
// confined to the active block; y = y_fwd + y_rev. A commit of the finished
// block runs the same forward chain and keeps its last state as the new cache.
//
// A step of one sequence with D = 1536 channels has only 48 rows, so one CTA
// per row leaves most SMs idle and the step's time is the length of each
// warp's instruction stream: its 32 tokens form a dependency chain. The
// kernel therefore gives every lane one state (16 warps per CTA) and keeps
// that stream short:
//   * each token's decay a = 2^(delta A log2 e) and input b = delta x B are
//     formed once and kept in registers for both chains (no second read of
//     delta x and B, no second multiply);
//   * B and C are widened into a state-major fp32 layout [N][T], so a warp
//     (one state) reads four tokens' values with one 16-byte broadcast load;
//   * the forward chain (from the cache) and the block-confined reverse chain
//     (from zero) run interleaved: two independent dependency chains per lane.
// The state arithmetic is that of every other kernel (decay_input and
// scan_step at one state per lane), so a committed cache has the bits of a
// one-shot prefill's boundary state; the 16 per-state partials of a token's
// output are added in state order 0..15.
#pragma once

#include "bdscan_kernels.cuh"

namespace bdk {

// Channel widths of a CTA: 32 channels with one state per warp (16 warps), or
// 16 channels with two states per warp (8 warps: lanes 0-15 hold state 2w and
// lanes 16-31 state 2w+1 of the same 16 channels) when even 16-channel rows
// leave SMs idle -- twice the SMs share the block's exps, and a token's output
// is still a sum inside one CTA.
template <int CW>
struct StepCfg {
    static constexpr int N = 16;
    static constexpr int SPW = 32 / CW;          // states per warp
    static constexpr int NW = N / SPW;           // warps per CTA
    static constexpr int THREADS = 32 * NW;
    static_assert(CW == 32 || CW == 16, "channel width");
};

// Shared-memory carve-up (bytes; every offset is a multiple of 16). T = staged
// tokens (the block length when known at compile time, else 32).
template <class IO, int T, int CW>
struct StepLayout {
    using CF = StepCfg<CW>;
    static constexpr int N = 16;
    static constexpr int TP = CF::SPW > 1 ? T + 4 : T;     // state-major row (padded: the two states of a warp in other banks)
    static constexpr int xb = T * CW * (int)sizeof(IO);    // one x / dt / z tile [T][CW]
    static constexpr int bb = T * N * (int)sizeof(IO);     // one B / C tile [T][N]
    static constexpr int xs = 0, dts = xs + xb, zs = dts + xb, Bs = zs + xb, Cs = Bs + bb;
    static constexpr int dd = Cs + bb;                     // float2 (delta, delta x) [T][CW]
    static constexpr int bt = dd + T * CW * 8;             // float B, state-major [N][TP]
    static constexpr int ct = bt + N * TP * 4;             // float C, state-major [N][TP]
    static constexpr int red = ct + N * TP * 4;            // float2 partials [warps][T/2][32 lanes]
    static constexpr int bytes = red + CF::NW * (T / 2) * 32 * 8;
    static_assert(xb % 16 == 0 && bb % 16 == 0 && T % 4 == 0, "16-byte rows, 4-token loads");
};

// KC = block length when fixed at compile time (4, 16 or 32), or 0 for a
// runtime block length of at most 32 tokens. The call covers exactly one block
// (L == K). h0 = the cache (read only); h_out = where the state after the block
// goes (a commit: the cache itself, in place), or null. CW = channels per CTA.
template <class IO, int KC, int CW>
__global__ void __launch_bounds__(StepCfg<CW>::THREADS, 1) bdscan_step_kernel(const ScanArgs a) {
    using CF = StepCfg<CW>;
    constexpr int N = 16, SPW = CF::SPW, NT = CF::THREADS;
    constexpr int T = KC > 0 ? KC : 32;
    using LY = StepLayout<IO, T, CW>;
    constexpr int TP = LY::TP;

    extern __shared__ __align__(16) char smem[];
    const IO *xs = reinterpret_cast<const IO *>(smem + LY::xs);
    const IO *zs = reinterpret_cast<const IO *>(smem + LY::zs);
    float2 *dd = reinterpret_cast<float2 *>(smem + LY::dd);
    float *Bt = reinterpret_cast<float *>(smem + LY::bt);
    float *Ct = reinterpret_cast<float *>(smem + LY::ct);
    float2 *red = reinterpret_cast<float2 *>(smem + LY::red);

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int cl = lane % CW;                     // this lane's channel in the tile
    const int n = warp * SPW + lane / CW;         // this lane's state
    const int64_t b = blockIdx.y;
    const int64_t d0 = (int64_t)blockIdx.x * CW;
    const int64_t d = d0 + cl;
    const bool dvalid = d < a.D;
    const int K = KC > 0 ? KC : a.K;   // tokens of the block (== L)
    const bool gated = a.z != nullptr;

    // Programmatic dependent launch: let the next kernel of the stream start
    // launching, and wait for the previous one (its memory visible) before the
    // first global access.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---- stage the block: x, dt, z [K][CW channels], B and C [K][N]
    {
        constexpr int EPC = 16 / (int)sizeof(IO);   // elements per 16-byte chunk
        constexpr int XC = CW / EPC;                // chunks per x row
        constexpr int BC = N / EPC;                 // chunks per B row
        const int64_t row0 = b * a.L;
        IO *sx = reinterpret_cast<IO *>(smem + LY::xs);
        IO *sdt = reinterpret_cast<IO *>(smem + LY::dts);
        IO *sz = reinterpret_cast<IO *>(smem + LY::zs);
        IO *sB = reinterpret_cast<IO *>(smem + LY::Bs);
        IO *sC = reinterpret_cast<IO *>(smem + LY::Cs);
        for (int e = tid; e < T * XC; e += NT) {
            const int t = e / XC, ch = e % XC;
            const int64_t dc = d0 + (int64_t)ch * EPC;
            const bool ok = t < K && dc < a.D;
            const int64_t off = ok ? ((row0 + t) * a.D + dc) : 0;
            const int so = t * CW + ch * EPC;
            cp_async16(sx + so, static_cast<const IO *>(a.x) + off, ok);
            cp_async16(sdt + so, static_cast<const IO *>(a.dt) + off, ok);
            if (gated) cp_async16(sz + so, static_cast<const IO *>(a.z) + off, ok);
        }
        for (int e = tid; e < T * BC; e += NT) {
            const int t = e / BC, ch = e % BC;
            const bool ok = t < K;
            const int64_t off = ok ? ((row0 + t) * N + (int64_t)ch * EPC) : 0;
            const int so = t * N + ch * EPC;
            cp_async16(sB + so, static_cast<const IO *>(a.B) + off, ok);
            cp_async16(sC + so, static_cast<const IO *>(a.C) + off, ok);
        }
        cp_async_commit();
    }

    // per-lane constants (global loads in flight with the copies); this
    // thread's readout item: token pair q, channel cr
    const int q = tid / CW, cr = tid % CW;   // (T/2) * CW <= threads
    const int64_t dr_ = d0 + cr;
    const float dfac = dr_ < a.D ? __fmul_rn(2.f, a.Dskip[dr_]) : 0.f;
    const float al = dvalid ? __fmul_rn(a.A[d * N + n], kLog2e) : 0.f;
    const float h = (dvalid && a.h0) ? a.h0[(b * a.D + d) * N + n] : 0.f;

    cp_async_wait<0>();
    __syncthreads();
    // ---- delta, delta x once per (token, channel); B, C to fp32, state-major
    {
        const IO *sdt = reinterpret_cast<const IO *>(smem + LY::dts);
        for (int e = tid; e < T * CW; e += NT) {
            const float xv = to_f32(xs[e]);
            const float dr = to_f32(sdt[e]);
            const float dl = a.dt_softplus ? softplus_f32(dr) : dr;
            dd[e] = make_float2(dl, __fmul_rn(dl, xv));
        }
        const IO *sB = reinterpret_cast<const IO *>(smem + LY::Bs);
        const IO *sC = reinterpret_cast<const IO *>(smem + LY::Cs);
        for (int e = tid; e < T * N; e += NT) {
            const int t = e % T, ns = e / T;   // consecutive threads: consecutive tokens of one state
            Bt[ns * TP + t] = to_f32(sB[t * N + ns]);
            Ct[ns * TP + t] = to_f32(sC[t * N + ns]);
        }
    }
    __syncthreads();

    // ---- decays and inputs of every token
    const float2 *ddc = dd + cl;
    const float4 *B4 = reinterpret_cast<const float4 *>(Bt + n * TP);   // [T/4]; one address per state
    const float4 *C4 = reinterpret_cast<const float4 *>(Ct + n * TP);
    const float al1[1] = {al};
    float at[T][1], bq[T][1], yp[T];
#pragma unroll
    for (int t4 = 0; t4 < T / 4; ++t4) {
        const float4 bv = B4[t4];
        const float bs[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int t = 4 * t4 + k;
            const float2 dv = (KC > 0 || t < K) ? ddc[t * CW] : make_float2(0.f, 0.f);
            decay_input<1>(al1, dv, bs + k, at[t], bq[t]);
        }
    }
    // ---- the forward chain (from the cache) and the reverse chain (from zero):
    // interleaved when the block length is known, else one after the other.
    // yp[t] = (forward partial) + (reverse partial), a sum of exactly two terms.
    float hs[1] = {h}, gs[1] = {0.f};
    if constexpr (KC > 0) {
#pragma unroll
        for (int i4 = 0; i4 < T / 4; ++i4) {
            const float4 cf4 = C4[i4], cr4 = C4[T / 4 - 1 - i4];
            const float cfs[4] = {cf4.x, cf4.y, cf4.z, cf4.w};
            const float crs[4] = {cr4.w, cr4.z, cr4.y, cr4.x};   // tokens T-1-4*i4-k
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int i = 4 * i4 + k, tf = i, tr = T - 1 - i;
                const float vf = scan_step<1>(hs, at[tf], bq[tf], cfs + k);
                const float vr = scan_step<1>(gs, at[tr], bq[tr], crs + k);
                if (i < T / 2) {
                    yp[tf] = vf;
                    yp[tr] = vr;
                } else {
                    yp[tf] = __fadd_rn(yp[tf], vf);
                    yp[tr] = __fadd_rn(yp[tr], vr);
                }
            }
        }
    } else {
#pragma unroll
        for (int t4 = 0; t4 < T / 4; ++t4) {
            const float4 cv = C4[t4];
            const float cs[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int t = 4 * t4 + k;
                if (t < K) yp[t] = scan_step<1>(hs, at[t], bq[t], cs + k);
            }
        }
#pragma unroll
        for (int t4 = T / 4 - 1; t4 >= 0; --t4) {
            const float4 cv = C4[t4];
            const float cs[4] = {cv.x, cv.y, cv.z, cv.w};
#pragma unroll
            for (int k = 3; k >= 0; --k) {
                const int t = 4 * t4 + k;
                if (t < K) yp[t] = __fadd_rn(yp[t], scan_step<1>(gs, at[t], bq[t], cs + k));
            }
        }
    }

    // ---- readout: partials [warp][token pair][lane] as float2; thread (q, c)
    // then adds the 16 states' partials of token pair q, channel c in state
    // order (state m: warp m / SPW, lane (m % SPW) * CW + c)
    {
        float2 *wrow = red + warp * (T / 2) * 32 + lane;
#pragma unroll
        for (int q = 0; q < T / 2; ++q) wrow[q * 32] = make_float2(yp[2 * q], yp[2 * q + 1]);
    }
    __syncthreads();
    if (q < T / 2 && 2 * q < K) {
        const float2 *src = red + q * 32 + cr;
        float2 ys = make_float2(0.f, 0.f);
#pragma unroll
        for (int m = 0; m < N; ++m) ys = __fadd2_rn(ys, src[(m / SPW) * (T / 2) * 32 + (m % SPW) * CW]);
        if (a.y && dr_ < a.D) {
            IO *gy = static_cast<IO *>(a.y) + (b * a.L) * a.D + dr_;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int t = 2 * q + k;
                if (t < K) {
                    float v = __fmaf_rn(dfac, to_f32(xs[t * CW + cr]), k == 0 ? ys.x : ys.y);
                    if (gated) v = __fmul_rn(v, silu_f32(to_f32(zs[t * CW + cr])));
                    IO o;
                    from_f32(v, o);
                    gy[(int64_t)t * a.D] = o;
                }
            }
        }
    }
    if (a.h_out && dvalid) a.h_out[(b * a.D + d) * N + n] = hs[0];
}

}  // namespace bdk
