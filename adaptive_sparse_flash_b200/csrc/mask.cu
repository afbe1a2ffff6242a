// mask.cu - transposed copy of the bit-packed block mask, for the key-block-parallel backward.
//
// The forward writes mask[bh][I][J / 32] (bit J % 32: key block J is nonzero for query block I); the
// dK/dV pass walks key block J's query blocks with find-first-set over maskT[bh][J][I / 32]
// (AdaSplash-2, gist.science (de), "Bit-Packed Block Mask", 32 blocks per 32-bit word).
#include <cuda_runtime.h>
#include <stdint.h>

#include "launch.h"

namespace eattn {
namespace {

// One thread per output word: gathers 32 query blocks' bits for one key block.
__global__ void mask_transpose_kernel(const uint32_t* __restrict__ mask, uint32_t* __restrict__ maskT, int nqb,
                                      int nkb, int nw, int nwq) {
    const int bh = blockIdx.y;
    const int t = blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= nkb * nwq) return;
    const int J = t / nwq;
    const int iw = t % nwq;
    const uint32_t* m = mask + (size_t)bh * nqb * nw;
    uint32_t out = 0u;
    const int i0 = iw * 32;
    const int i1 = min(nqb, i0 + 32);
    for (int I = i0; I < i1; ++I) out |= ((m[(size_t)I * nw + (J >> 5)] >> (J & 31)) & 1u) << (I - i0);
    maskT[(size_t)bh * nkb * nwq + t] = out;
}

}  // namespace

cudaError_t launch_mask_transpose(const uint32_t* mask, uint32_t* maskT, int BH, int nqb, int nkb, int nw, int nwq,
                                  cudaStream_t stream) {
    const int words = nkb * nwq;
    dim3 grid((words + 255) / 256, BH);
    launch_mark(stream);
    mask_transpose_kernel<<<grid, 256, 0, stream>>>(mask, maskT, nqb, nkb, nw, nwq);
    return cudaGetLastError();
}

}  // namespace eattn
