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

constexpr int kStepWarps = 16;                 // one warp per state (N = 16)
constexpr int kStepThreads = 32 * kStepWarps;  // 512

// Shared-memory carve-up (bytes; every offset is a multiple of 16). T = staged
// tokens (the block length when known at compile time, else 32).
template <class IO, int T>
struct StepLayout {
    static constexpr int N = 16;
    static constexpr int xb = T * kCh * (int)sizeof(IO);   // one x / dt / z tile [T][32]
    static constexpr int bb = T * N * (int)sizeof(IO);     // one B / C tile [T][N]
    static constexpr int xs = 0, dts = xs + xb, zs = dts + xb, Bs = zs + xb, Cs = Bs + bb;
    static constexpr int dd = Cs + bb;                     // float2 (delta, delta x) [T][32]
    static constexpr int bt = dd + T * kCh * 8;            // float B, state-major [N][T]
    static constexpr int ct = bt + N * T * 4;              // float C, state-major [N][T]
    static constexpr int red = ct + N * T * 4;             // float2 partials [16 warps][T/2][32]
    static constexpr int bytes = red + kStepWarps * (T / 2) * kCh * 8;
    static_assert(xb % 16 == 0 && bb % 16 == 0 && T % 4 == 0, "16-byte rows, 4-token loads");
};

// KC = block length when fixed at compile time (4, 16 or 32), or 0 for a
// runtime block length of at most 32 tokens. The call covers exactly one block
// (L == K). h0 = the cache (read only); h_out = where the state after the block
// goes (a commit: the cache itself, in place), or null.
template <class IO, int KC>
__global__ void __launch_bounds__(kStepThreads, 1) bdscan_step_kernel(const ScanArgs a) {
    constexpr int N = 16;
    constexpr int T = KC > 0 ? KC : 32;
    using LY = StepLayout<IO, T>;

    extern __shared__ __align__(16) char smem[];
    const IO *xs = reinterpret_cast<const IO *>(smem + LY::xs);
    const IO *zs = reinterpret_cast<const IO *>(smem + LY::zs);
    float2 *dd = reinterpret_cast<float2 *>(smem + LY::dd);
    float *Bt = reinterpret_cast<float *>(smem + LY::bt);
    float *Ct = reinterpret_cast<float *>(smem + LY::ct);
    float2 *red = reinterpret_cast<float2 *>(smem + LY::red);

    const int tid = threadIdx.x, c = tid & 31, warp = tid >> 5;   // warp = this lane's state
    const int64_t b = blockIdx.y;
    const int64_t d0 = (int64_t)blockIdx.x * kCh;
    const int64_t d = d0 + c;
    const bool dvalid = d < a.D;
    const int K = KC > 0 ? KC : a.K;   // tokens of the block (== L)
    const bool gated = a.z != nullptr;

    // Programmatic dependent launch: let the next kernel of the stream start
    // launching, and wait for the previous one (its memory visible) before the
    // first global access.
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    asm volatile("griddepcontrol.wait;" ::: "memory");

    // ---- stage the block: x, dt, z [K][32 channels], B and C [K][N]
    {
        constexpr int EPC = 16 / (int)sizeof(IO);   // elements per 16-byte chunk
        constexpr int XC = kCh / EPC;               // chunks per x row
        constexpr int BC = N / EPC;                 // chunks per B row
        const int64_t row0 = b * a.L;
        IO *sx = reinterpret_cast<IO *>(smem + LY::xs);
        IO *sdt = reinterpret_cast<IO *>(smem + LY::dts);
        IO *sz = reinterpret_cast<IO *>(smem + LY::zs);
        IO *sB = reinterpret_cast<IO *>(smem + LY::Bs);
        IO *sC = reinterpret_cast<IO *>(smem + LY::Cs);
        for (int e = tid; e < T * XC; e += kStepThreads) {
            const int t = e / XC, ch = e % XC;
            const int64_t dc = d0 + (int64_t)ch * EPC;
            const bool ok = t < K && dc < a.D;
            const int64_t off = ok ? ((row0 + t) * a.D + dc) : 0;
            const int so = t * kCh + ch * EPC;
            cp_async16(sx + so, static_cast<const IO *>(a.x) + off, ok);
            cp_async16(sdt + so, static_cast<const IO *>(a.dt) + off, ok);
            if (gated) cp_async16(sz + so, static_cast<const IO *>(a.z) + off, ok);
        }
        for (int e = tid; e < T * BC; e += kStepThreads) {
            const int t = e / BC, ch = e % BC;
            const bool ok = t < K;
            const int64_t off = ok ? ((row0 + t) * N + (int64_t)ch * EPC) : 0;
            const int so = t * N + ch * EPC;
            cp_async16(sB + so, static_cast<const IO *>(a.B) + off, ok);
            cp_async16(sC + so, static_cast<const IO *>(a.C) + off, ok);
        }
        cp_async_commit();
    }

    // per-lane constants (global loads in flight with the copies)
    const float dskip = dvalid ? a.Dskip[d] : 0.f;
    const float dfac = __fmul_rn(2.f, dskip);
    const float al = dvalid ? __fmul_rn(a.A[d * N + warp], kLog2e) : 0.f;
    const float h = (dvalid && a.h0) ? a.h0[(b * a.D + d) * N + warp] : 0.f;

    cp_async_wait<0>();
    __syncthreads();
    // ---- delta, delta x once per (token, channel); B, C to fp32, state-major
    {
        const IO *sdt = reinterpret_cast<const IO *>(smem + LY::dts);
        for (int e = tid; e < T * kCh; e += kStepThreads) {
            const float xv = to_f32(xs[e]);
            const float dr = to_f32(sdt[e]);
            const float dl = a.dt_softplus ? softplus_f32(dr) : dr;
            dd[e] = make_float2(dl, __fmul_rn(dl, xv));
        }
        const IO *sB = reinterpret_cast<const IO *>(smem + LY::Bs);
        const IO *sC = reinterpret_cast<const IO *>(smem + LY::Cs);
        for (int e = tid; e < T * N; e += kStepThreads) {
            const int t = e % T, n = e / T;   // consecutive threads: consecutive tokens of one state
            Bt[e] = to_f32(sB[t * N + n]);
            Ct[e] = to_f32(sC[t * N + n]);
        }
    }
    __syncthreads();

    // ---- decays and inputs of every token
    const float2 *ddc = dd + c;
    const float4 *B4 = reinterpret_cast<const float4 *>(Bt + warp * T);   // [T/4], same address in every lane
    const float4 *C4 = reinterpret_cast<const float4 *>(Ct + warp * T);
    const float al1[1] = {al};
    float at[T][1], bq[T][1], yp[T];
#pragma unroll
    for (int t4 = 0; t4 < T / 4; ++t4) {
        const float4 bv = B4[t4];
        const float bs[4] = {bv.x, bv.y, bv.z, bv.w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int t = 4 * t4 + k;
            const float2 dv = (KC > 0 || t < K) ? ddc[t * kCh] : make_float2(0.f, 0.f);
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

    // ---- readout: partials [warp][token pair][channel] as float2; warp w then
    // adds the 16 states' partials of token pair w in state order
    {
        float2 *wrow = red + warp * (T / 2) * kCh + c;
#pragma unroll
        for (int q = 0; q < T / 2; ++q) wrow[q * kCh] = make_float2(yp[2 * q], yp[2 * q + 1]);
    }
    __syncthreads();
    const int q = warp;
    if (q < T / 2 && 2 * q < K) {
        const float2 *src = red + q * kCh + c;
        float2 ys = make_float2(0.f, 0.f);
#pragma unroll
        for (int s = 0; s < kStepWarps; ++s) ys = __fadd2_rn(ys, src[s * (T / 2) * kCh]);
        if (a.y && dvalid) {
            IO *gy = static_cast<IO *>(a.y) + (b * a.L) * a.D + d;
#pragma unroll
            for (int k = 0; k < 2; ++k) {
                const int t = 2 * q + k;
                if (t < K) {
                    float v = __fmaf_rn(dfac, to_f32(xs[t * kCh + c]), k == 0 ? ys.x : ys.y);
                    if (gated) v = __fmul_rn(v, silu_f32(to_f32(zs[t * kCh + c])));
                    IO o;
                    from_f32(v, o);
                    gy[(int64_t)t * a.D] = o;
                }
            }
        }
    }
    if (a.h_out && dvalid) a.h_out[(b * a.D + d) * N + warp] = hs[0];
}

}  // namespace bdk
