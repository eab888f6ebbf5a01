// Compiled fast path of the Python binding for the calls a denoising loop makes
// once per step: bdscan_block_step and bdscan_commit_block (and a prepared
// block step). Argument marshalling only, like bdscan.py: the common case --
// CUDA tensors of the expected dtype, shape and contiguity, all on one device --
// is recognised here with direct tensor accessors, the C-ABI structs are filled
// on the stack and the entry point is called on PyTorch's current stream.
// Anything else returns kNotCommon without touching the library, so the Python
// binding runs its own checks and raises the specific error. The status the
// library returns is passed back unchanged.
#include <torch/extension.h>
#include <c10/cuda/CUDAStream.h>

#include <tuple>

#include "bdscan.h"

namespace {

constexpr int64_t kNotCommon = -1;

bool io_ok(const at::Tensor &t, at::ScalarType io, const c10::Device &dev, c10::IntArrayRef shape) {
    return t.defined() && t.scalar_type() == io && t.device() == dev && t.sizes() == shape && t.is_contiguous();
}

struct Call {
    bdscan_dims dims;
    bdscan_inputs ins;
};

// The tests of the Python binding's common path over x, dt, A, B, C, Dskip, z.
bool prepare(const at::Tensor &x, const at::Tensor &dt, const at::Tensor &A, const at::Tensor &B,
             const at::Tensor &C, const at::Tensor &Dskip, const c10::optional<at::Tensor> &z, bool dt_softplus,
             Call &c) {
    if (!x.defined() || x.dim() != 3 || !x.is_cuda() || !x.is_contiguous() || !B.defined() || B.dim() != 3)
        return false;
    const at::ScalarType io = x.scalar_type();
    if (io != at::kFloat && io != at::kBFloat16) return false;
    const int64_t Bt = x.size(0), L = x.size(1), D = x.size(2), N = B.size(2);
    const c10::Device dev = x.device();
    const int64_t bs[3] = {Bt, L, N}, an[2] = {D, N}, dn[1] = {D};
    if (!io_ok(dt, io, dev, x.sizes()) || !io_ok(B, io, dev, bs) || !io_ok(C, io, dev, bs) ||
        !io_ok(A, at::kFloat, dev, an) || !io_ok(Dskip, at::kFloat, dev, dn))
        return false;
    if (z.has_value() && !io_ok(*z, io, dev, x.sizes())) return false;
    c.dims = bdscan_dims{Bt, L, D, N, L, io == at::kBFloat16 ? BDSCAN_BF16 : BDSCAN_F32, dt_softplus ? 1 : 0};
    c.ins = bdscan_inputs{x.data_ptr(), dt.data_ptr(), B.data_ptr(), C.data_ptr(),
                          z.has_value() ? z->data_ptr() : nullptr, A.data_ptr<float>(), Dskip.data_ptr<float>()};
    return true;
}

bdscan_stream_t current_stream(const at::Tensor &x) {
    return reinterpret_cast<bdscan_stream_t>(c10::cuda::getCurrentCUDAStream(x.device().index()).stream());
}

// y: the caller's tensor (checked) or a new one like x.
bool output(const at::Tensor &x, const c10::optional<at::Tensor> &y_in, at::Tensor &y) {
    if (y_in.has_value()) {
        if (!io_ok(*y_in, x.scalar_type(), x.device(), x.sizes())) return false;
        y = *y_in;
    } else {
        y = at::empty(x.sizes(), x.options());
    }
    return true;
}

// (status, y); status kNotCommon: not the common case, nothing was queued.
std::tuple<int64_t, at::Tensor> block_step(const at::Tensor &x, const at::Tensor &dt, const at::Tensor &A,
                                           const at::Tensor &B, const at::Tensor &C, const at::Tensor &Dskip,
                                           const at::Tensor &h_cache, const c10::optional<at::Tensor> &z,
                                           bool dt_softplus, const c10::optional<at::Tensor> &y_in) {
    Call c;
    at::Tensor y;
    if (!prepare(x, dt, A, B, C, Dskip, z, dt_softplus, c)) return {kNotCommon, y};
    const int64_t hs[3] = {c.dims.batch, c.dims.d_inner, c.dims.d_state};
    if (!io_ok(h_cache, at::kFloat, x.device(), hs) || !output(x, y_in, y)) return {kNotCommon, at::Tensor()};
    const int rc = bdscan_block_step(&c.dims, &c.ins, h_cache.data_ptr<float>(), y.data_ptr(), current_stream(x));
    return {rc, y};
}

// (status, y or undefined); h_cache is advanced in place.
std::tuple<int64_t, at::Tensor> commit_block(const at::Tensor &x, const at::Tensor &dt, const at::Tensor &A,
                                             const at::Tensor &B, const at::Tensor &C, const at::Tensor &Dskip,
                                             const at::Tensor &h_cache, const c10::optional<at::Tensor> &z,
                                             bool dt_softplus, bool want_y, const c10::optional<at::Tensor> &y_in) {
    Call c;
    at::Tensor y;
    if (!prepare(x, dt, A, B, C, Dskip, z, dt_softplus, c)) return {kNotCommon, y};
    const int64_t hs[3] = {c.dims.batch, c.dims.d_inner, c.dims.d_state};
    if (!io_ok(h_cache, at::kFloat, x.device(), hs)) return {kNotCommon, y};
    if ((want_y || y_in.has_value()) && !output(x, y_in, y)) return {kNotCommon, at::Tensor()};
    const int rc = bdscan_commit_block(&c.dims, &c.ins, h_cache.data_ptr<float>(), y.defined() ? y.data_ptr() : nullptr,
                                       current_stream(x));
    return {rc, y};
}

// A block step whose A, Dskip and cache were checked when it was prepared: the
// step's own tensors are checked against the prepared shape and device.
std::tuple<int64_t, at::Tensor> prepared_step(const at::Tensor &x, const at::Tensor &dt, const at::Tensor &B,
                                              const at::Tensor &C, const c10::optional<at::Tensor> &z,
                                              const c10::optional<at::Tensor> &y_in, int64_t batch, int64_t block,
                                              int64_t d_inner, int64_t d_state, bool bf16, bool dt_softplus,
                                              int64_t A_ptr, int64_t Dskip_ptr, int64_t h_ptr) {
    const at::ScalarType io = bf16 ? at::kBFloat16 : at::kFloat;
    if (!x.defined() || !x.is_cuda()) return {kNotCommon, at::Tensor()};
    const c10::Device dev = x.device();
    const int64_t xs[3] = {batch, block, d_inner}, bs[3] = {batch, block, d_state};
    if (!io_ok(x, io, dev, xs) || !io_ok(dt, io, dev, xs) || !io_ok(B, io, dev, bs) || !io_ok(C, io, dev, bs))
        return {kNotCommon, at::Tensor()};
    if (z.has_value() && !io_ok(*z, io, dev, xs)) return {kNotCommon, at::Tensor()};
    at::Tensor y;
    if (!output(x, y_in, y)) return {kNotCommon, at::Tensor()};
    const bdscan_dims dims{batch, block, d_inner, d_state, block, bf16 ? BDSCAN_BF16 : BDSCAN_F32, dt_softplus ? 1 : 0};
    const bdscan_inputs ins{x.data_ptr(), dt.data_ptr(), B.data_ptr(), C.data_ptr(),
                            z.has_value() ? z->data_ptr() : nullptr, reinterpret_cast<const float *>(A_ptr),
                            reinterpret_cast<const float *>(Dskip_ptr)};
    const int rc = bdscan_block_step(&dims, &ins, reinterpret_cast<const float *>(h_ptr), y.data_ptr(),
                                     current_stream(x));
    return {rc, y};
}

}  // namespace

PYBIND11_MODULE(TORCH_EXTENSION_NAME, m) {
    m.doc() = "compiled per-step marshalling for bdscan_block_step / bdscan_commit_block";
    m.def("block_step", &block_step);
    m.def("commit_block", &commit_block);
    m.def("prepared_step", &prepared_step);
    m.attr("NOT_COMMON") = kNotCommon;
}
