// C ABI of the block-confined bidirectional selective scan (see include/bdscan.h).
// Host side: argument checks, mode / template selection and launches.
#include <atomic>
#include <cstdint>
#include <mutex>

#include "../../include/bdscan.h"
#include "bdscan_backward.cuh"
#include "bdscan_backward16.cuh"
#include "bdscan_kernels.cuh"
#include "bdscan_lag.cuh"
#include "bdscan_step.cuh"

namespace {

thread_local cudaError_t g_last_cuda = cudaSuccess;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

enum Op { kTrain, kPrefill, kStep, kCommit, kCleanStream, kReverseAccumulate };
// kCleanStream: prefill with h_out optional; kReverseAccumulate: whole-sequence reverse scan added into y

int check_common(const bdscan_dims *dm, const bdscan_inputs *in) {
    if (!dm || !in) return BDSCAN_ERR_INVALID_ARG;
    if (dm->batch < 0 || dm->seqlen < 0 || dm->d_inner < 0 || dm->block < 1) return BDSCAN_ERR_INVALID_ARG;
    if (dm->io_dtype != BDSCAN_F32 && dm->io_dtype != BDSCAN_BF16) return BDSCAN_ERR_INVALID_ARG;
    if (dm->dt_softplus != 0 && dm->dt_softplus != 1) return BDSCAN_ERR_INVALID_ARG;
    if (dm->seqlen % dm->block != 0) return BDSCAN_ERR_INVALID_ARG;
    if (dm->d_state != 16 && dm->d_state != 64) return BDSCAN_ERR_UNSUPPORTED;
    if (dm->block > INT32_MAX) return BDSCAN_ERR_UNSUPPORTED;
    if (dm->batch > 65535) return BDSCAN_ERR_UNSUPPORTED;
    const int64_t vec = dm->io_dtype == BDSCAN_BF16 ? 8 : 4;
    if (dm->d_inner % vec != 0) return BDSCAN_ERR_UNSUPPORTED;
    // a pointer may be NULL only when its tensor has no elements
    const bool tok = dm->batch * dm->seqlen > 0;
    if (tok && dm->d_inner > 0 && (!in->x || !in->dt)) return BDSCAN_ERR_INVALID_ARG;
    if (tok && (!in->B || !in->C)) return BDSCAN_ERR_INVALID_ARG;
    if (dm->d_inner > 0 && (!in->A || !in->Dskip)) return BDSCAN_ERR_INVALID_ARG;
    const void *ptrs[] = {in->x, in->dt, in->B, in->C, in->z, in->A, in->Dskip};
    for (const void *p : ptrs)
        if (p && !aligned16(p)) return BDSCAN_ERR_ALIGNMENT;
    return BDSCAN_OK;
}

// dynamic shared memory a CTA may opt in to on sm_100 (227 KB), less room for the
// kernels' static shared memory
constexpr int kMaxDynSmem = 226 * 1024;

// span checkpoints of the long fused path: (spans - 1) x N states x 32 channels, fp32
size_t long_fused_ck_bytes(int64_t K, int N) {
    const int64_t spans = (K + bdk::kSpanLong - 1) / bdk::kSpanLong;
    return (size_t)(spans - 1) * (size_t)N * bdk::kCh * 4;
}

// (measured on the 4-states-per-lane layout, the larger one: the 8-state kernel
// that runs at N = 64 takes the same blocks)
template <class IO, int N>
bool long_fused_fits(int64_t K) {
    return bdk::Layout<IO, N, bdk::kLongFused, 0>::base_bytes + long_fused_ck_bytes(K, N) <= (size_t)kMaxDynSmem;
}

// Raise a kernel's dynamic shared-memory ceiling to cap bytes, once per device
// (mask: the kernel's own record of the devices already done).
template <class Kern>
int smem_ceiling_once(Kern kern, int cap, std::atomic<uint64_t> &mask) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(mask.load(std::memory_order_acquire) & bit)) {
        const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, cap);
        if (e != cudaSuccess) { g_last_cuda = e; return BDSCAN_ERR_CUDA; }
        mask.fetch_or(bit, std::memory_order_acq_rel);
    }
    return BDSCAN_OK;
}

// Launch kern(a) on st. pdl: with programmatic stream serialisation, so that the
// kernel's launch overlaps the end of the previous kernel in the stream (the
// kernel waits for it before touching global memory).
template <class Kern>
int launch_kernel(Kern kern, dim3 grid, int threads, size_t smem, cudaStream_t st, bool pdl,
                  const bdk::ScanArgs &a) {
    if (pdl) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = grid;
        cfg.blockDim = dim3(threads);
        cfg.dynamicSmemBytes = smem;
        cfg.stream = st;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attr[0].val.programmaticStreamSerializationAllowed = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        const cudaError_t le = cudaLaunchKernelEx(&cfg, kern, a);
        if (le != cudaSuccess) { (void)cudaGetLastError(); g_last_cuda = le; return BDSCAN_ERR_CUDA; }
    } else {
        kern<<<grid, threads, smem, st>>>(a);
    }
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) { g_last_cuda = e; return BDSCAN_ERR_CUDA; }
    return BDSCAN_OK;
}

// The fused, forward-only and long-block modes (bdscan_kernel).
template <class IO, int N, int MODE, int KC, int NPTV = 4>
int launch(const bdk::ScanArgs &a, int64_t batch, cudaStream_t st, unsigned gz = 1, bool pdl = false) {
    using CF = bdk::Cfg<N, MODE, KC, NPTV>;
    using LY = bdk::Layout<IO, N, MODE, KC, NPTV>;
    const size_t smem = LY::base_bytes + (MODE == bdk::kLong ? (size_t)a.K * bdk::kCh * 4
                                          : MODE == bdk::kLongFused ? long_fused_ck_bytes(a.K, N) : 0);
    auto kern = bdk::bdscan_kernel<IO, N, MODE, KC, NPTV>;
    static std::atomic<uint64_t> done_mask{0};
    const int cap = MODE == bdk::kLongFused ? kMaxDynSmem : LY::base_bytes + (MODE == bdk::kLong ? bdk::kLongSmemMax : 0);
    const int rc = smem_ceiling_once(kern, cap, done_mask);
    if (rc != BDSCAN_OK) return rc;
    const dim3 grid((unsigned)((a.D + bdk::kCh - 1) / bdk::kCh), (unsigned)batch, gz);
    return launch_kernel(kern, grid, CF::THREADS, smem, st, pdl, a);
}

// The lagged whole-block pass (bdscan_lag_kernel).
template <class IO, int N, int KC, int NPT>
int launch_lag(const bdk::ScanArgs &a, int64_t batch, cudaStream_t st) {
    using CF = bdk::LagCfg<N, KC, NPT>;
    using LY = bdk::LagLayout<IO, N, KC, NPT>;
    auto kern = bdk::bdscan_lag_kernel<IO, N, KC, NPT>;
    static std::atomic<uint64_t> done_mask{0};
    const int rc = smem_ceiling_once(kern, LY::bytes, done_mask);
    if (rc != BDSCAN_OK) return rc;
    const dim3 grid((unsigned)((a.D + bdk::kCh - 1) / bdk::kCh), (unsigned)batch, 1);
    return launch_kernel(kern, grid, CF::THREADS, LY::bytes, st, false, a);
}

// A block step (or a commit with y) of few rows at N = 16 (bdscan_step_kernel),
// CW channels per CTA.
template <class IO, int KC, int CW>
int launch_step(const bdk::ScanArgs &a, int64_t batch, cudaStream_t st, bool pdl) {
    constexpr int T = KC > 0 ? KC : 32;
    constexpr int smem = bdk::StepLayout<IO, T, CW>::bytes;
    auto kern = bdk::bdscan_step_kernel<IO, KC, CW>;
    static std::atomic<uint64_t> done_mask{0};
    const int rc = smem_ceiling_once(kern, smem, done_mask);
    if (rc != BDSCAN_OK) return rc;
    const dim3 grid((unsigned)((a.D + CW - 1) / CW), (unsigned)batch, 1);
    return launch_kernel(kern, grid, bdk::StepCfg<CW>::THREADS, smem, st, pdl, a);
}

int device_sm_count();

template <class IO, int N>
int dispatch_mode(int mode, const bdk::ScanArgs &a, int64_t batch, cudaStream_t st, unsigned gz = 1,
                  bool thin = false, bool pdl = false) {
    if constexpr (N == 16) {
        if (thin && mode == bdk::kFused) {   // one state per lane: the latency-bound small block step
            // 16-channel CTAs when even those leave no SM with two of them
            const bool half = batch * ((a.D + 15) / 16) <= device_sm_count();
            switch (a.K) {
                case 4: return half ? launch_step<IO, 4, 16>(a, batch, st, pdl) : launch_step<IO, 4, 32>(a, batch, st, pdl);
                case 16: return half ? launch_step<IO, 16, 16>(a, batch, st, pdl) : launch_step<IO, 16, 32>(a, batch, st, pdl);
                case 32: return half ? launch_step<IO, 32, 16>(a, batch, st, pdl) : launch_step<IO, 32, 32>(a, batch, st, pdl);
                default: return half ? launch_step<IO, 0, 16>(a, batch, st, pdl) : launch_step<IO, 0, 32>(a, batch, st, pdl);
            }
        }
    }
    // several whole blocks of 16 or 32 tokens: the lagged schedule (the reverse
    // chain one block behind the forward chain). Blocks of 4 keep the phased
    // kernel: their 4-step phases are too short to carry the lag (measured
    // 8.8 -> 10.2 ms per 350M-stack layer).
    if (mode == bdk::kFused && !thin && a.L >= 2 * (int64_t)a.K) {
        if constexpr (N == 16) {
            if (a.K == 16) return launch_lag<IO, N, 16, 4>(a, batch, st);
            if (a.K == 32) return launch_lag<IO, N, 32, 4>(a, batch, st);
        } else {
            if (a.K == 16) return launch_lag<IO, N, 16, 8>(a, batch, st);
        }
    }
    if constexpr (N == 64) {
        if (mode == bdk::kFused) {   // 8 states per lane where a whole block fits TMEM
            if (a.K == 4) return launch<IO, N, bdk::kFused, 4, 8>(a, batch, st, 1, pdl);
            if (a.K == 16) return launch<IO, N, bdk::kFused, 16, 8>(a, batch, st, 1, pdl);
        }
    }
    if (mode == bdk::kForwardOnly) return launch<IO, N, bdk::kForwardOnly, 0>(a, batch, st, gz, pdl);
    if (mode == bdk::kLong) return launch<IO, N, bdk::kLong, 0>(a, batch, st, 1, pdl);
    if (mode == bdk::kLongFused) {
        if constexpr (N == 64)   // 8 states per lane: a span's a, b fill the SM's TMEM
            return launch<IO, N, bdk::kLongFused, 0, 8>(a, batch, st, 1, pdl);
        else
            return launch<IO, N, bdk::kLongFused, 0>(a, batch, st, 1, pdl);
    }
    if (mode == bdk::kReverseAcc) return launch<IO, N, bdk::kReverseAcc, 0>(a, batch, st, 1, pdl);
    switch (a.K) {
        case 4: return launch<IO, N, bdk::kFused, 4>(a, batch, st, 1, pdl);
        case 16: return launch<IO, N, bdk::kFused, 16>(a, batch, st, 1, pdl);
        case 32: return launch<IO, N, bdk::kFused, 32>(a, batch, st, 1, pdl);
        default: return launch<IO, N, bdk::kFused, 0>(a, batch, st, 1, pdl);
    }
}

struct Chunking {   // time-chunked prefill: chunk length, chunk count, pass, workspace halves
    int64_t len = 0, count = 1;
    int pass = 0;
    float *ws_h = nullptr, *ws_p = nullptr;
};

// Number of SMs of the current device, queried once per device.
int device_sm_count() {
    static std::atomic<int> sms[64] = {};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    int n = sms[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
        sms[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

// Every argument check of one pass, and the kernel mode it selects; queues
// nothing. Multi-pass entry points call this for all their passes before the
// first launch, so a call that returns an error has queued no work.
int validate(Op op, const bdscan_dims *dm, const bdscan_inputs *in, const float *h0, const void *y,
             const float *h_out, const float *boundary, int *mode_out) {
    int rc = check_common(dm, in);
    if (rc != BDSCAN_OK) return rc;
    if ((op == kStep || op == kCommit) && dm->seqlen != dm->block) return BDSCAN_ERR_INVALID_ARG;
    const bool any_y = dm->batch * dm->seqlen * dm->d_inner > 0;
    const bool any_state = dm->batch * dm->d_inner > 0;
    if ((op == kTrain || op == kStep || op == kReverseAccumulate) && any_y && !y) return BDSCAN_ERR_INVALID_ARG;
    if ((op == kPrefill || op == kCommit) && any_state && !h_out) return BDSCAN_ERR_INVALID_ARG;
    if (op == kStep && any_state && !h0) return BDSCAN_ERR_INVALID_ARG;
    const void *outs[] = {h0, y, h_out, boundary};
    for (const void *p : outs)
        if (p && !aligned16(p)) return BDSCAN_ERR_ALIGNMENT;

    int mode;
    if (op == kReverseAccumulate) {
        mode = bdk::kReverseAcc;
    } else if (op == kPrefill || op == kCleanStream || (op == kCommit && !y)) {
        mode = bdk::kForwardOnly;
    } else if (dm->block <= 32) {
        mode = bdk::kFused;
    } else {
        const bool bf = dm->io_dtype == BDSCAN_BF16;
        const bool fits = dm->d_state == 16 ? (bf ? long_fused_fits<__nv_bfloat16, 16>(dm->block)
                                                  : long_fused_fits<float, 16>(dm->block))
                                            : (bf ? long_fused_fits<__nv_bfloat16, 64>(dm->block)
                                                  : long_fused_fits<float, 64>(dm->block));
        if (fits && dm->seqlen < (int64_t(1) << 30)) {   // (its tile schedule counts steps in 32 bits)
            mode = bdk::kLongFused;
        } else {
            if (dm->block * bdk::kCh * 4 > bdk::kLongSmemMax) return BDSCAN_ERR_UNSUPPORTED;
            mode = bdk::kLong;
        }
    }
    if (mode_out) *mode_out = mode;
    return BDSCAN_OK;
}

int run(Op op, const bdscan_dims *dm, const bdscan_inputs *in, const float *h0, void *y, float *h_out,
        float *boundary, bdscan_stream_t stream, const float *blk_h0 = nullptr, const Chunking *ch = nullptr) {
    int mode = 0;
    const int rc = validate(op, dm, in, h0, y, h_out, boundary, &mode);
    if (rc != BDSCAN_OK) return rc;
    if (dm->batch == 0 || dm->d_inner == 0) return BDSCAN_OK;   // nothing to compute or write

    bdk::ScanArgs a;
    a.x = in->x; a.dt = in->dt; a.B = in->B; a.C = in->C; a.z = in->z;
    a.A = in->A; a.Dskip = in->Dskip; a.h0 = h0;
    a.y = y; a.h_out = h_out; a.boundary = boundary; a.blk_h0 = blk_h0;
    a.chunk_len = ch ? ch->len : 0;
    a.chunk_pass = ch ? ch->pass : 0;
    a.ws_h = ch ? ch->ws_h : nullptr;
    a.ws_p = ch ? ch->ws_p : nullptr;
    const unsigned gz = ch ? (unsigned)ch->count : 1u;
    a.L = dm->seqlen; a.D = dm->d_inner; a.K = (int32_t)dm->block; a.dt_softplus = dm->dt_softplus;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // a block step (or a commit with y) of at most one (batch, 32-channel) row
    // per SM runs bdscan_step_kernel (one state per lane)
    bool thin = false;
    if ((op == kStep || (op == kCommit && y)) && mode == bdk::kFused && dm->d_state == 16)
        thin = dm->batch * ((dm->d_inner + bdk::kCh - 1) / bdk::kCh) <= device_sm_count();
    // block steps and commits are short, back-to-back launches: overlap each
    // one's launch with the end of the kernel before it
    const bool pdl = op == kStep || op == kCommit;
    if (dm->io_dtype == BDSCAN_BF16)
        return dm->d_state == 16 ? dispatch_mode<__nv_bfloat16, 16>(mode, a, dm->batch, st, gz, thin, pdl)
                                 : dispatch_mode<__nv_bfloat16, 64>(mode, a, dm->batch, st, gz, false, pdl);
    return dm->d_state == 16 ? dispatch_mode<float, 16>(mode, a, dm->batch, st, gz, thin, pdl)
                             : dispatch_mode<float, 64>(mode, a, dm->batch, st, gz, false, pdl);
}

// Resident CTAs per SM of the forward-only scan kernel (both passes of the
// time-chunked prefill run it), queried once per device; without a device the
// value the kernels reach on sm_100 (3 at N = 16, 1 at N = 64).
template <class IO, int N>
int forward_only_ctas_per_sm() {
    static std::atomic<int> cache[64] = {};
    const int fallback = N == 16 ? 3 : 1;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return fallback;
    int n = cache[dev].load(std::memory_order_relaxed);
    if (n == 0) {
        using CF = bdk::Cfg<N, bdk::kForwardOnly, 0>;
        using LY = bdk::Layout<IO, N, bdk::kForwardOnly, 0>;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, bdk::bdscan_kernel<IO, N, bdk::kForwardOnly, 0>,
                                                          CF::THREADS, LY::base_bytes) != cudaSuccess || n <= 0) {
            (void)cudaGetLastError();
            n = fallback;
        }
        cache[dev].store(n, std::memory_order_relaxed);
    }
    return n;
}

int forward_only_slots(const bdscan_dims *dm) {
    const int per_sm = dm->io_dtype == BDSCAN_BF16
                           ? (dm->d_state == 16 ? forward_only_ctas_per_sm<__nv_bfloat16, 16>()
                                                : forward_only_ctas_per_sm<__nv_bfloat16, 64>())
                           : (dm->d_state == 16 ? forward_only_ctas_per_sm<float, 16>()
                                                : forward_only_ctas_per_sm<float, 64>());
    return per_sm * device_sm_count();
}

// Chunk plan of the time-chunked prefill. Chunks cost a second pass, so they
// are used only when the (batch, 32-channel) rows alone give fewer CTAs than
// the device has SMs; then as many chunks as keep all CTAs resident in one
// wave (rows x chunks <= SMs x resident CTAs per SM: a second, partial wave
// would nearly double the time), at most 64 chunks and at least 256 tokens per
// chunk. The chunk length is a multiple of 16 tokens.
Chunking chunk_plan(const bdscan_dims *dm) {
    Chunking c;
    const int sms = device_sm_count();
    const int64_t row_ctas = dm->batch * ((dm->d_inner + bdk::kCh - 1) / bdk::kCh);
    int64_t g = (row_ctas > 0 && row_ctas < sms) ? forward_only_slots(dm) / row_ctas : 1;
    const int64_t gmax_len = dm->seqlen / 256 > 0 ? dm->seqlen / 256 : 1;
    if (g > 64) g = 64;
    if (g > gmax_len) g = gmax_len;
    if (g < 1) g = 1;
    int64_t len = (dm->seqlen + g - 1) / g;
    len = ((len + 15) / 16) * 16;
    if (len < 16) len = 16;
    c.len = len;
    c.count = (dm->seqlen + len - 1) / len;
    if (c.count < 1) c.count = 1;
    return c;
}

size_t chunked_ws_bytes(const bdscan_dims *dm, const Chunking &c) {
    if (c.count <= 1) return 0;
    return 2 * (size_t)dm->batch * (size_t)c.count * (size_t)dm->d_inner * (size_t)dm->d_state * sizeof(float);
}

// Argument checks of both passes of the time-chunked prefill (queues nothing).
int check_chunked_passes(const bdscan_dims *dm, const bdscan_inputs *in, const float *h0, const void *y,
                         const float *h_out, const float *boundary) {
    const int rc = validate(kCleanStream, dm, in, nullptr, nullptr, nullptr, nullptr, nullptr);
    return rc != BDSCAN_OK ? rc : validate(kPrefill, dm, in, h0, y, h_out, boundary, nullptr);
}

// The two passes of the time-chunked prefill on caller-provided scratch
// (ws: 2 * batch * chunks * D * N floats, 16-byte aligned).
int prefill_chunked_on(const bdscan_dims *dm, const bdscan_inputs *in, const float *h0, void *y, float *h_out,
                       float *boundary, float *ws, bdscan_stream_t stream) {
    Chunking c = chunk_plan(dm);
    if (c.count <= 1)   // enough parallelism without chunks: the sequential scan (bit-identical caches)
        return run(kPrefill, dm, in, h0, y, h_out, boundary, stream);
    // both passes' checks before the first launch (pass 2 alone needs h_out, y, boundary)
    int rc = check_chunked_passes(dm, in, h0, y, h_out, boundary);
    if (rc != BDSCAN_OK) return rc;
    const size_t half = (size_t)dm->batch * c.count * dm->d_inner * dm->d_state;
    c.ws_h = ws;
    c.ws_p = ws + half;
    c.pass = 1;
    rc = run(kCleanStream, dm, in, nullptr, nullptr, nullptr, nullptr, stream, nullptr, &c);
    if (rc != BDSCAN_OK) return rc;
    c.pass = 2;
    return run(kPrefill, dm, in, h0, y, h_out, boundary, stream, nullptr, &c);
}

// ---- backward pass of the all-block training scan ------------------------------
struct BwdPlan {
    int64_t ct, ntb, nck;
    size_t bc, a, d, ck;   // float counts of the workspace regions (each a multiple of 4)
};

size_t round4(size_t v) { return (v + 3) & ~(size_t)3; }

BwdPlan bwd_plan(const bdscan_dims *dm) {
    BwdPlan p;
    const int TT = dm->d_state == 16 ? bdk::BwdCfg<16>::TT : bdk::BwdCfg<64>::TT;   // tokens per tile
    p.ct = (dm->d_inner + bdk::kCh - 1) / bdk::kCh;
    p.ntb = dm->block > TT ? (dm->block + TT - 1) / TT : 1;
    p.nck = p.ntb > 2 ? p.ntb - 2 : 0;
    p.bc = round4((size_t)dm->batch * p.ct * dm->seqlen * 2 * dm->d_state);
    p.a = round4((size_t)dm->batch * dm->d_inner * dm->d_state);
    p.d = round4((size_t)dm->batch * dm->d_inner);
    p.ck = (size_t)dm->batch * p.ct * p.nck * (dm->d_state / 4) * bdk::kCh * 8;
    return p;
}

size_t bwd_ws_bytes(const BwdPlan &p) { return (p.bc + p.a + p.d + p.ck) * sizeof(float); }

template <class IO, int N>
int launch_bwd(const bdk::BwdArgs &a, int64_t batch, int64_t ct, void *dB, void *dC, float *dA, float *dDskip,
               cudaStream_t st) {
    using CF = bdk::BwdCfg<N>;
    using LY = bdk::BwdLayout<IO, N>;
    // blocks of 16 at N = 16: each block staged once (bdscan_bwd16_kernel)
    const bool b16 = N == 16 && a.K == 16;
    auto kern = b16 ? bdk::bdscan_bwd16_kernel<IO> : bdk::bdscan_bwd_kernel<IO, N>;
    const int smem = b16 ? bdk::Bwd16Layout<IO>::bytes : LY::bytes;
    static std::atomic<uint64_t> mask16{0}, mask_tiles{0};   // per kernel
    const int rc = smem_ceiling_once(kern, smem, b16 ? mask16 : mask_tiles);
    if (rc != BDSCAN_OK) return rc;
    if (batch > 0 && ct > 0) {
        kern<<<dim3((unsigned)ct, (unsigned)batch), CF::THREADS, smem, st>>>(a);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) { g_last_cuda = e; return BDSCAN_ERR_CUDA; }
    }
    const int64_t total = batch * a.L * 2 * N + a.D * N + a.D;
    if (total > 0) {
        int64_t blocks = (total + 255) / 256;
        if (blocks > 148 * 16) blocks = 148 * 16;
        bdk::bdscan_bwd_reduce<IO, N><<<(unsigned)blocks, 256, 0, st>>>(a.ws_bc, a.ws_a, a.ws_d, dB, dC, dA, dDskip,
                                                                        batch, a.L, a.D, ct);
        cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) { g_last_cuda = e; return BDSCAN_ERR_CUDA; }
    }
    return BDSCAN_OK;
}

// ---- context-parallel pieces: the fold of gathered chunk summaries ------------
// h_in = P_{r-1} (... (P_0 h0 + H_0) ...) + H_{r-1}: the forward state at the
// start of chunk r, from the (H, P) summaries of chunks 0 .. r-1 ([chunks][count]).
__global__ void __launch_bounds__(256) bdscan_carry_fold_kernel(const float *__restrict__ h0,
                                                                const float *__restrict__ H,
                                                                const float *__restrict__ P, int64_t count,
                                                                int64_t upto, float *__restrict__ h_in) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
        float h = h0 ? h0[i] : 0.f;
        for (int64_t q = 0; q < upto; ++q) h = __fmaf_rn(P[q * count + i], h, H[q * count + i]);
        h_in[i] = h;
    }
}

// the summary of an empty context: H = 0, P = 1
__global__ void __launch_bounds__(256) bdscan_identity_summary_kernel(float *H, float *P, int64_t count) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
        H[i] = 0.f;
        P[i] = 1.f;
    }
}

unsigned elementwise_blocks(int64_t count) {
    int64_t blocks = (count + 255) / 256;
    if (blocks > 148 * 8) blocks = 148 * 8;
    return (unsigned)(blocks > 0 ? blocks : 1);
}

// ---- allocation-free variant of the time-chunked prefill -----------------------
// Scratch for bdscan_prefill_chunked_noalloc: a fixed array in device global
// memory, created when the library is loaded on a device and kept until the
// process exits. 2^21 floats = 8 MiB per device.
constexpr size_t kStaticScratchFloats = size_t(1) << 21;
static __device__ __align__(256) float g_prefill_scratch[kStaticScratchFloats];

// Device address of g_prefill_scratch, looked up once per device. In host code
// the symbol name is only a handle; cudaGetSymbolAddress turns it into the
// address the kernels must be given.
float *static_scratch_address(int *err) {
    static std::mutex mu;
    static float *addr[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= 64) {
        *err = e != cudaSuccess ? (int)e : (int)cudaErrorInvalidDevice;
        return nullptr;
    }
    std::lock_guard<std::mutex> lock(mu);
    if (!addr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_prefill_scratch);
        if (e != cudaSuccess) {
            *err = (int)e;
            return nullptr;
        }
        addr[dev] = static_cast<float *>(p);
    }
    *err = 0;
    return addr[dev];
}

}  // namespace

extern "C" {

int bdscan_prefill_chunked_noalloc(const bdscan_dims *dims, const bdscan_inputs *in, const float *h0, void *y,
                                   float *h_out, float *boundary, bdscan_stream_t stream) {
    int rc = check_chunked_passes(dims, in, h0, y, h_out, boundary);
    if (rc != BDSCAN_OK) return rc;
    const size_t need = chunked_ws_bytes(dims, chunk_plan(dims));
    if (need > kStaticScratchFloats * sizeof(float)) return BDSCAN_ERR_WORKSPACE;   // beyond the fixed scratch
    float *ws = nullptr;
    if (need > 0) {
        int err = 0;
        ws = static_scratch_address(&err);
        if (!ws) {
            g_last_cuda = static_cast<cudaError_t>(err);
            return BDSCAN_ERR_CUDA;
        }
    }
    // pass 1 writes every scratch entry that pass 2 reads, so nothing needs clearing
    return prefill_chunked_on(dims, in, h0, y, h_out, boundary, ws, stream);
}

size_t bdscan_prefill_chunked_workspace(const bdscan_dims *dims) {
    if (!dims || dims->batch < 0 || dims->seqlen < 0 || dims->d_inner < 0 || dims->d_state < 0) return 0;
    return chunked_ws_bytes(dims, chunk_plan(dims));
}

int bdscan_prefill_chunked(const bdscan_dims *dims, const bdscan_inputs *in, const float *h0, void *y,
                           float *h_out, float *boundary, void *ws, size_t ws_bytes, bdscan_stream_t stream) {
    int rc = check_common(dims, in);
    if (rc != BDSCAN_OK) return rc;
    const size_t need = chunked_ws_bytes(dims, chunk_plan(dims));
    if (need > 0 && (!ws || ws_bytes < need)) return BDSCAN_ERR_WORKSPACE;
    if (ws && !aligned16(ws)) return BDSCAN_ERR_ALIGNMENT;
    return prefill_chunked_on(dims, in, h0, y, h_out, boundary, static_cast<float *>(ws), stream);
}

size_t bdscan_train_blocks_backward_workspace(const bdscan_dims *dims) {
    if (!dims || dims->batch < 0 || dims->seqlen < 0 || dims->d_inner < 0 || dims->block < 1) return 0;
    if (dims->d_state != 16 && dims->d_state != 64) return 0;
    return bwd_ws_bytes(bwd_plan(dims));
}

int bdscan_train_blocks_backward(const bdscan_dims *dims, const bdscan_inputs *in, const float *h0,
                                 const float *boundary, const void *dy, const bdscan_grads *gr, void *ws,
                                 size_t ws_bytes, bdscan_stream_t stream) {
    int rc = check_common(dims, in);
    if (rc != BDSCAN_OK) return rc;
    if (!gr) return BDSCAN_ERR_INVALID_ARG;
    const bdscan_dims *dm = dims;
    const bool tok = dm->batch * dm->seqlen > 0;
    const bool elems = tok && dm->d_inner > 0;
    if (elems && (!dy || !gr->dx || !gr->ddt)) return BDSCAN_ERR_INVALID_ARG;
    if (elems && in->z && !gr->dz) return BDSCAN_ERR_INVALID_ARG;
    if (tok && (!gr->dB || !gr->dC)) return BDSCAN_ERR_INVALID_ARG;
    if (dm->d_inner > 0 && (!gr->dA || !gr->dDskip)) return BDSCAN_ERR_INVALID_ARG;
    if (elems && dm->seqlen > dm->block && !boundary) return BDSCAN_ERR_INVALID_ARG;
    if (dm->batch > 65535) return BDSCAN_ERR_UNSUPPORTED;
    const void *al[] = {dy, gr->dx, gr->ddt, gr->dz, gr->dB, gr->dC};
    for (const void *p : al)
        if (p && !aligned16(p)) return BDSCAN_ERR_ALIGNMENT;
    const BwdPlan p = bwd_plan(dm);
    const size_t need = bwd_ws_bytes(p);
    if (need > 0 && (!ws || ws_bytes < need)) return BDSCAN_ERR_WORKSPACE;
    if (ws && !aligned16(ws)) return BDSCAN_ERR_ALIGNMENT;
    if (dm->d_inner == 0) return BDSCAN_OK;
    bdk::BwdArgs a{};
    a.x = in->x; a.dt = in->dt; a.B = in->B; a.C = in->C; a.z = in->z; a.dy = dy;
    a.A = in->A; a.Dskip = in->Dskip; a.h0 = h0; a.boundary = boundary;
    a.dx = gr->dx; a.ddt = gr->ddt; a.dz = gr->dz; a.dh0 = gr->dh0;
    float *w = static_cast<float *>(ws);
    a.ws_bc = w;
    a.ws_a = w + p.bc;
    a.ws_d = a.ws_a + p.a;
    a.ws_ck = p.ck ? a.ws_d + p.d : nullptr;
    a.L = dm->seqlen; a.D = dm->d_inner; a.nck = p.nck;
    a.K = (int32_t)dm->block; a.dt_softplus = dm->dt_softplus;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dm->io_dtype == BDSCAN_BF16)
        return dm->d_state == 16 ? launch_bwd<__nv_bfloat16, 16>(a, dm->batch, p.ct, gr->dB, gr->dC, gr->dA, gr->dDskip, st)
                                 : launch_bwd<__nv_bfloat16, 64>(a, dm->batch, p.ct, gr->dB, gr->dC, gr->dA, gr->dDskip, st);
    return dm->d_state == 16 ? launch_bwd<float, 16>(a, dm->batch, p.ct, gr->dB, gr->dC, gr->dA, gr->dDskip, st)
                             : launch_bwd<float, 64>(a, dm->batch, p.ct, gr->dB, gr->dC, gr->dA, gr->dDskip, st);
}

int bdscan_chunk_summary(const bdscan_dims *dims, const bdscan_inputs *in, float *H, float *P,
                         bdscan_stream_t stream) {
    int rc = check_common(dims, in);
    if (rc != BDSCAN_OK) return rc;
    const int64_t count = dims->batch * dims->d_inner * dims->d_state;
    if (count == 0) return BDSCAN_OK;
    if (!H || !P) return BDSCAN_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dims->seqlen == 0) {
        bdscan_identity_summary_kernel<<<elementwise_blocks(count), 256, 0, st>>>(H, P, count);
        const cudaError_t e = cudaGetLastError();
        if (e != cudaSuccess) { g_last_cuda = e; return BDSCAN_ERR_CUDA; }
        return BDSCAN_OK;
    }
    // the first pass of the time-chunked prefill, over one chunk: the whole context
    Chunking c;
    c.len = dims->seqlen;
    c.count = 1;
    c.pass = 1;
    c.ws_h = H;
    c.ws_p = P;
    return run(kCleanStream, dims, in, nullptr, nullptr, nullptr, nullptr, stream, nullptr, &c);
}

int bdscan_carry_fold(int64_t chunks, int64_t index, int64_t count, const float *h0, const float *H_all,
                      const float *P_all, float *h_in, bdscan_stream_t stream) {
    if (chunks < 1 || index < 0 || index >= chunks || count < 0) return BDSCAN_ERR_INVALID_ARG;
    if (count == 0) return BDSCAN_OK;
    if (!h_in || (index > 0 && (!H_all || !P_all))) return BDSCAN_ERR_INVALID_ARG;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    bdscan_carry_fold_kernel<<<elementwise_blocks(count), 256, 0, st>>>(h0, H_all, P_all, count, index, h_in);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) { g_last_cuda = e; return BDSCAN_ERR_CUDA; }
    return BDSCAN_OK;
}

int bdscan_train_blocks(const bdscan_dims *dims, const bdscan_inputs *in, const float *h0, void *y,
                        float *boundary, float *h_out, bdscan_stream_t stream) {
    return run(kTrain, dims, in, h0, y, h_out, boundary, stream);
}

int bdscan_prefill(const bdscan_dims *dims, const bdscan_inputs *in, const float *h0, void *y, float *h_out,
                   float *boundary, bdscan_stream_t stream) {
    return run(kPrefill, dims, in, h0, y, h_out, boundary, stream);
}

int bdscan_block_step(const bdscan_dims *dims, const bdscan_inputs *in, const float *h_cache, void *y,
                      bdscan_stream_t stream) {
    return run(kStep, dims, in, h_cache, y, nullptr, nullptr, stream);
}

int bdscan_commit_block(const bdscan_dims *dims, const bdscan_inputs *in, float *h_cache, void *y,
                        bdscan_stream_t stream) {
    return run(kCommit, dims, in, h_cache, y, h_cache, nullptr, stream);
}

int bdscan_train_two_stream(const bdscan_dims *dims, const bdscan_inputs *clean, const bdscan_inputs *noisy,
                            const float *h0, void *y_clean, void *y_noisy, float *boundary, float *h_out,
                            bdscan_stream_t stream) {
    int rc = check_common(dims, noisy);
    if (rc != BDSCAN_OK) return rc;
    rc = check_common(dims, clean);
    if (rc != BDSCAN_OK) return rc;
    const bool any_block = dims->batch * dims->d_inner > 0 && dims->seqlen > 0;
    if (any_block && !boundary) return BDSCAN_ERR_INVALID_ARG;
    // both passes' checks (y_noisy, the long-block mode) before the first launch
    rc = validate(kCleanStream, dims, clean, h0, y_clean, h_out, boundary, nullptr);
    if (rc == BDSCAN_OK) rc = validate(kTrain, dims, noisy, h0, y_noisy, nullptr, nullptr, nullptr);
    if (rc != BDSCAN_OK) return rc;
    // the clean stream: forward-only scan writing the block caches (and y_clean)
    rc = run(kCleanStream, dims, clean, h0, y_clean, h_out, boundary, stream);
    if (rc != BDSCAN_OK) return rc;
    // the noisy stream: every block restarts from the clean cache at its start
    return run(kTrain, dims, noisy, h0, y_noisy, nullptr, nullptr, stream, boundary);
}

int bdscan_full_bidirectional(const bdscan_dims *dims, const bdscan_inputs *in, const float *h0, void *y,
                              float *h_out, bdscan_stream_t stream) {
    if (!dims || !in) return BDSCAN_ERR_INVALID_ARG;
    bdscan_inputs ungated = *in;
    ungated.z = nullptr;
    // both passes' checks (y is required by the second) before the first launch
    int rc = validate(kCleanStream, dims, &ungated, h0, y, h_out, nullptr, nullptr);
    if (rc == BDSCAN_OK) rc = validate(kReverseAccumulate, dims, in, nullptr, y, nullptr, nullptr, nullptr);
    if (rc != BDSCAN_OK) return rc;
    // forward pass: y = y_fwd + Dskip x (ungated)
    rc = run(kCleanStream, dims, &ungated, h0, y, h_out, nullptr, stream);
    if (rc != BDSCAN_OK) return rc;
    // reverse pass over the whole sequence: y = (y + y_rev + Dskip x) * gate
    return run(kReverseAccumulate, dims, in, nullptr, y, nullptr, nullptr, stream);
}

const char *bdscan_status_string(int status) {
    switch (status) {
        case BDSCAN_OK: return "BDSCAN_OK";
        case BDSCAN_ERR_INVALID_ARG: return "BDSCAN_ERR_INVALID_ARG";
        case BDSCAN_ERR_UNSUPPORTED: return "BDSCAN_ERR_UNSUPPORTED";
        case BDSCAN_ERR_ALIGNMENT: return "BDSCAN_ERR_ALIGNMENT";
        case BDSCAN_ERR_WORKSPACE: return "BDSCAN_ERR_WORKSPACE";
        case BDSCAN_ERR_CUDA: return "BDSCAN_ERR_CUDA";
        default: return "BDSCAN_UNKNOWN_STATUS";
    }
}

const char *bdscan_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda); }

int bdscan_version(void) { return 100; }

}  // extern "C"
