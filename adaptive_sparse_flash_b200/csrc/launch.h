// launch.h - host launchers implemented by the kernel files (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fwd_common.cuh"

namespace eattn {

// Records the caller's next timing event (entmax_opts.events) on `stream`, if the current API call was given
// any; every launcher calls it right before each kernel launch (api.cu).
void launch_mark(cudaStream_t stream);

// fp16 operand copies (f16.cu): `count` bf16 tensors of n16 16-byte chunks each; maxbits[t] receives
// max |x| of tensor t as float bits.
struct F16Job {
    const void* src[4];
    void* dst[4];
    uint32_t* maxbits;
    size_t n16;
    int count;
};
cudaError_t launch_to_f16(const F16Job& job, int num_sms, cudaStream_t stream);

// Power-of-two exponent e >= 0 by which a tensor with max |x| = maxbits (float bits) is scaled down in
// its fp16 copy: 0 while the max is below 2^15, else exponent(max) - 14.
__host__ __device__ inline int f16_range_exp(uint32_t maxbits) {
    const int E = (int)((maxbits >> 23) & 0xffu) - 127;
    return E >= 15 ? E - 14 : 0;
}

cudaError_t launch_fwd_simt(const FwdArgs& a, bool fp32, cudaStream_t stream);
cudaError_t launch_fwd_h(const FwdArgs& a, cudaStream_t stream);
size_t fwd_h_smem_bytes(int nw, int bins);
cudaError_t launch_fwd_tc(const FwdArgs& a, cudaStream_t stream);
size_t fwd_tc_smem_bytes(int d, int nw);
size_t fwd_simt_smem_bytes(int d, int nkb, int mb, int nw);
cudaError_t make_tmap_bf16(CUtensorMap* map, const void* base, int BH, int n, int d, int rows);
cudaError_t make_tmap_f16(CUtensorMap* map, const void* base, int BH, int n, int d, int rows);

// maskT[bh][J][I / 32] bit I % 32 = mask[bh][I][J / 32] bit J % 32
cudaError_t launch_mask_transpose(const uint32_t* mask, uint32_t* maskT, int BH, int nqb, int nkb, int nw, int nwq,
                                  cudaStream_t stream);

struct BwdArgs {
    const void* Q;
    const void* K;
    const void* V;
    const void* O;
    const void* dO;
    const float* rowstat;   // entmax: tau; softmax: lse (natural log)
    const uint32_t* mask;   // [BH][nqb][nw], nullptr: dense (causal) traversal
    const uint32_t* maskT;  // [BH][nkb][nwq], nullptr: dense
    const float* obar;      // entmax: U V fp32 [BH][n][d]
    const float* sum_u;     // entmax: [BH][n]
    void* dQ;
    void* dK;
    void* dV;
    int* status;
    int B, H, n, d;
    int nqb, nkb, nw, nwq;
    int causal;
    int softmax;            // 1: softmax baseline, 0: entmax
    float scale;
    float cz;               // entmax: (alpha - 1) * scale
    float k;                // entmax: 1 / (alpha - 1)
    int kind;               // entmax AlphaKind
    // fp16 path (bwd_h.cu): copies of Q, K, V (from the forward) and dO, and their range exponents
    const void* Qh;
    const void* Kh;
    const void* Vh;
    const void* dOh;
    const uint32_t* maxbits;  // [4]: Q, K, V, dO
};

cudaError_t launch_bwd(const BwdArgs& a, float* delta_pad, float* stat_pad, cudaStream_t stream);
cudaError_t launch_bwd_pre(const BwdArgs& a, float* delta_pad, float* stat_pad, cudaStream_t stream);
cudaError_t launch_bwd_h(const BwdArgs& a, float* delta_pad, float* stat_pad, cudaStream_t stream);
size_t bwd_smem_bytes(int d, int nw, int nwq);

struct SoftmaxFwdArgs {
    const void* Q;
    const void* K;
    const void* V;
    void* O;
    float* lse;
    int* status;
    int B, H, n, d, causal, ntiles;
    float scale;
    // fp16 path (softmax_fwd_h.cu, d = 64): copies of Q, K, V and their range exponents
    const void* Qh;
    const void* Kh;
    const void* Vh;
    const uint32_t* maxbits;
};
cudaError_t launch_softmax_fwd(const SoftmaxFwdArgs& a, cudaStream_t stream);
cudaError_t launch_softmax_fwd_h(const SoftmaxFwdArgs& a, cudaStream_t stream);

}  // namespace eattn
