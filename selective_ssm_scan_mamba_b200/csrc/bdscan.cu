// C ABI of the block-confined bidirectional selective scan (see include/bdscan.h).
// Host side: argument checks, mode / template selection and launches.
#include <atomic>
#include <cstdint>

#include "../../include/bdscan.h"
#include "bdscan_kernels.cuh"

namespace {

thread_local cudaError_t g_last_cuda = cudaSuccess;

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

enum Op { kTrain, kPrefill, kStep, kCommit };

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

template <class IO, int N, int MODE, int KC>
int launch(const bdk::ScanArgs &a, int64_t batch, cudaStream_t st) {
    using CF = bdk::Cfg<N, MODE, KC>;
    using LY = bdk::Layout<IO, N, MODE, KC>;
    const size_t smem = LY::base_bytes + (MODE == bdk::kLong ? (size_t)a.K * bdk::kCh * 4 : 0);
    auto kern = bdk::bdscan_kernel<IO, N, MODE, KC>;
    // raise the dynamic shared-memory ceiling once per device
    static std::atomic<uint64_t> done_mask{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) dev = 0;
    const uint64_t bit = 1ull << (dev & 63);
    if (!(done_mask.load(std::memory_order_acquire) & bit)) {
        const int cap = LY::base_bytes + (MODE == bdk::kLong ? bdk::kLongSmemMax : 0);
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, cap);
        if (e != cudaSuccess) { g_last_cuda = e; return BDSCAN_ERR_CUDA; }
        done_mask.fetch_or(bit, std::memory_order_acq_rel);
    }
    dim3 grid((unsigned)((a.D + bdk::kCh - 1) / bdk::kCh), (unsigned)batch);
    kern<<<grid, CF::THREADS, smem, st>>>(a);
    const cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) { g_last_cuda = e; return BDSCAN_ERR_CUDA; }
    return BDSCAN_OK;
}

template <class IO, int N>
int dispatch_mode(int mode, const bdk::ScanArgs &a, int64_t batch, cudaStream_t st) {
    if (mode == bdk::kForwardOnly) return launch<IO, N, bdk::kForwardOnly, 0>(a, batch, st);
    if (mode == bdk::kLong) return launch<IO, N, bdk::kLong, 0>(a, batch, st);
    switch (a.K) {
        case 4: return launch<IO, N, bdk::kFused, 4>(a, batch, st);
        case 16: return launch<IO, N, bdk::kFused, 16>(a, batch, st);
        case 32: return launch<IO, N, bdk::kFused, 32>(a, batch, st);
        default: return launch<IO, N, bdk::kFused, 0>(a, batch, st);
    }
}

int run(Op op, const bdscan_dims *dm, const bdscan_inputs *in, const float *h0, void *y, float *h_out,
        float *boundary, bdscan_stream_t stream) {
    int rc = check_common(dm, in);
    if (rc != BDSCAN_OK) return rc;
    if ((op == kStep || op == kCommit) && dm->seqlen != dm->block) return BDSCAN_ERR_INVALID_ARG;
    const bool any_y = dm->batch * dm->seqlen * dm->d_inner > 0;
    const bool any_state = dm->batch * dm->d_inner > 0;
    if ((op == kTrain || op == kStep) && any_y && !y) return BDSCAN_ERR_INVALID_ARG;
    if ((op == kPrefill || op == kCommit) && any_state && !h_out) return BDSCAN_ERR_INVALID_ARG;
    if (op == kStep && any_state && !h0) return BDSCAN_ERR_INVALID_ARG;
    const void *outs[] = {h0, y, h_out, boundary};
    for (const void *p : outs)
        if (p && !aligned16(p)) return BDSCAN_ERR_ALIGNMENT;

    int mode;
    if (op == kPrefill || (op == kCommit && !y)) {
        mode = bdk::kForwardOnly;
    } else if (dm->block <= 32) {
        mode = bdk::kFused;
    } else {
        if (dm->block * bdk::kCh * 4 > bdk::kLongSmemMax) return BDSCAN_ERR_UNSUPPORTED;
        mode = bdk::kLong;
    }
    if (dm->batch == 0 || dm->d_inner == 0) return BDSCAN_OK;   // nothing to compute or write

    bdk::ScanArgs a;
    a.x = in->x; a.dt = in->dt; a.B = in->B; a.C = in->C; a.z = in->z;
    a.A = in->A; a.Dskip = in->Dskip; a.h0 = h0;
    a.y = y; a.h_out = h_out; a.boundary = boundary;
    a.L = dm->seqlen; a.D = dm->d_inner; a.K = (int32_t)dm->block; a.dt_softplus = dm->dt_softplus;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    if (dm->io_dtype == BDSCAN_BF16)
        return dm->d_state == 16 ? dispatch_mode<__nv_bfloat16, 16>(mode, a, dm->batch, st)
                                 : dispatch_mode<__nv_bfloat16, 64>(mode, a, dm->batch, st);
    return dm->d_state == 16 ? dispatch_mode<float, 16>(mode, a, dm->batch, st)
                             : dispatch_mode<float, 64>(mode, a, dm->batch, st);
}

}  // namespace

extern "C" {

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

const char *bdscan_status_string(int status) {
    switch (status) {
        case BDSCAN_OK: return "BDSCAN_OK";
        case BDSCAN_ERR_INVALID_ARG: return "BDSCAN_ERR_INVALID_ARG";
        case BDSCAN_ERR_UNSUPPORTED: return "BDSCAN_ERR_UNSUPPORTED";
        case BDSCAN_ERR_ALIGNMENT: return "BDSCAN_ERR_ALIGNMENT";
        case BDSCAN_ERR_CUDA: return "BDSCAN_ERR_CUDA";
        default: return "BDSCAN_UNKNOWN_STATUS";
    }
}

const char *bdscan_last_cuda_error(void) { return cudaGetErrorString(g_last_cuda); }

int bdscan_version(void) { return 100; }

}  // extern "C"
