// f16.cu - fp16 operand copies of bf16 tensors, with a per-tensor power-of-two range scale.
//
// The entmax kernels for alpha <= 2 feed the tensor cores fp16 operands: P and U lie in [0, 1], where
// fp16 keeps 11 significant bits against bf16's 8, so one fp16 product replaces a two-term bf16 split.
// Every bf16 value of magnitude in [2^-14, 2^15) converts to fp16 exactly. A tensor whose largest
// magnitude reaches 2^15 is stored scaled by 2^-e (e = exponent of the max - 14, so the scaled max stays
// below 2^15); the consumers multiply the products back by 2^e, which is exact.
//
// Pass 1 converts unscaled and records max |x| of each tensor (as float bits: non-negative floats order
// like their bit patterns). Pass 2 reconverts, scaled, only the tensors that need it; with every input
// in range its blocks exit at once.
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "launch.h"

namespace eattn {
namespace {

constexpr int kCvtThreads = 256;

__device__ __forceinline__ uint32_t cvt_word(uint32_t w, float s, float& mx) {
    const float lo = __uint_as_float(w << 16);
    const float hi = __uint_as_float(w & 0xffff0000u);
    mx = fmaxf(mx, fmaxf(fabsf(lo), fabsf(hi)));
    const __half2 h = __floats2half2_rn(lo * s, hi * s);
    return *reinterpret_cast<const uint32_t*>(&h);
}

__global__ void __launch_bounds__(kCvtThreads) to_f16_pass1(F16Job job) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (int t = 0; t < job.count; ++t) {
        const uint4* src = static_cast<const uint4*>(job.src[t]);
        uint4* dst = static_cast<uint4*>(job.dst[t]);
        float mx = 0.0f;
        for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < job.n16; i += stride) {
            const uint4 v = src[i];
            uint4 o;
            o.x = cvt_word(v.x, 1.0f, mx);
            o.y = cvt_word(v.y, 1.0f, mx);
            o.z = cvt_word(v.z, 1.0f, mx);
            o.w = cvt_word(v.w, 1.0f, mx);
            dst[i] = o;
        }
        // NaN compares false: a NaN input never raises the max (it stays a NaN in the copy, as in bf16)
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
        if ((threadIdx.x & 31) == 0 && mx > 0.0f) atomicMax(&job.maxbits[t], __float_as_uint(mx));
    }
}

__global__ void __launch_bounds__(kCvtThreads) to_f16_pass2(F16Job job) {
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    for (int t = 0; t < job.count; ++t) {
        const int e = f16_range_exp(job.maxbits[t]);
        if (e == 0) continue;
        const float s = __uint_as_float((uint32_t)(127 - e) << 23);  // 2^-e, e <= 114
        const uint4* src = static_cast<const uint4*>(job.src[t]);
        uint4* dst = static_cast<uint4*>(job.dst[t]);
        float mx = 0.0f;
        for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < job.n16; i += stride) {
            const uint4 v = src[i];
            uint4 o;
            o.x = cvt_word(v.x, s, mx);
            o.y = cvt_word(v.y, s, mx);
            o.z = cvt_word(v.z, s, mx);
            o.w = cvt_word(v.w, s, mx);
            dst[i] = o;
        }
    }
}

}  // namespace

cudaError_t launch_to_f16(const F16Job& job, int num_sms, cudaStream_t stream) {
    if (job.count < 1 || job.count > 4) return cudaErrorInvalidValue;
    cudaError_t e = cudaMemsetAsync(job.maxbits, 0, sizeof(uint32_t) * job.count, stream);
    if (e != cudaSuccess) return e;
    // memory-bound copy: 8 resident blocks of 256 threads per SM, grid-stride
    const size_t want = (job.n16 + kCvtThreads - 1) / kCvtThreads;
    const int grid1 = (int)(want < (size_t)num_sms * 8 ? (want > 0 ? want : 1) : (size_t)num_sms * 8);
    launch_mark(stream);
    to_f16_pass1<<<grid1, kCvtThreads, 0, stream>>>(job);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    launch_mark(stream);
    to_f16_pass2<<<num_sms, kCvtThreads, 0, stream>>>(job);
    return cudaGetLastError();
}

}  // namespace eattn
