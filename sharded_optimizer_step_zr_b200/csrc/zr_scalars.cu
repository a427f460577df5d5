// The AdamW scalars computed on the device, for steps whose count (and,
// optionally, learning rate) lives in device memory, so that a CUDA graph
// that captured the step replays as successive steps of a schedule.
#include <cuda_runtime.h>

#include <cstdint>

#include "zr_internal.hpp"

namespace zr {
namespace {

// One thread: advance the device step count and compute the AdamW scalars
// for the new step, in fp64 from the fp32 hyperparameters and rounded once
// to fp32 -- the same expressions as the host computes for zr_step.  The
// learning rate is read from d_lr when given (a schedule updated on the
// device), else it is hp.lr.
__global__ void zr_device_scalars_kernel(int64_t* d_step, const zr_adamw hp, const float* d_lr, AdamScalars* out) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    const int64_t step = *d_step + 1;
    *d_step = step;
    const float lr_f = d_lr != nullptr ? *d_lr : hp.lr;
    const double b1 = hp.beta1, b2 = hp.beta2, lr = lr_f, t = static_cast<double>(step);
    AdamScalars s;
    s.beta1 = hp.beta1;
    s.beta2 = hp.beta2;
    s.one_minus_beta1 = static_cast<float>(1.0 - b1);
    s.one_minus_beta2 = static_cast<float>(1.0 - b2);
    s.step_size = static_cast<float>(lr / (1.0 - pow(b1, t)));
    s.bc2_sqrt = static_cast<float>(sqrt(1.0 - pow(b2, t)));
    s.decay = static_cast<float>(1.0 - lr * static_cast<double>(hp.weight_decay));
    s.eps = hp.eps;
    *out = s;
}

}  // namespace

int launch_device_scalars(int64_t* d_step, const zr_adamw& hp, const float* d_lr, AdamScalars* out, void* stream_v) {
    zr_device_scalars_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream_v)>>>(d_step, hp, d_lr, out);
    return cudaGetLastError();
}

}  // namespace zr
