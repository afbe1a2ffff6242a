// api.cu - host side of the C ABI: argument validation, workspace layout, status word, launches.
//
// Nothing here allocates or frees device memory, and nothing synchronises except
// entmax_attn_check(). Every argument error returns before the first CUDA call.
#include <cuda.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "common.cuh"
#include "entmax_attn.h"
#include "fwd_common.cuh"
#include "launch.h"

namespace eattn {

__device__ int g_status;  // ENTMAX_OK, or the first device-side error since the last check

// Timing events of the API call running on this host thread (entmax_opts.events): event i is recorded right
// before the call's i-th kernel launch, and one more after its last launch.
namespace {
struct EventTrail {
    void* const* events = nullptr;
    int count = 0;
    int next = 0;
};
thread_local EventTrail t_trail;

// Installs the trail of one API call for its duration; the destructor records the closing event.
struct TrailScope {
    cudaStream_t stream;
    TrailScope(const entmax_opts* o, cudaStream_t s) : stream(s) {
        t_trail = EventTrail{};
        if (o && o->events && o->num_events > 0) {
            t_trail.events = o->events;
            t_trail.count = o->num_events;
        }
    }
    ~TrailScope() {
        launch_mark(stream);
        t_trail = EventTrail{};
    }
};
}  // namespace

void launch_mark(cudaStream_t stream) {
    if (t_trail.events && t_trail.next < t_trail.count) {
        cudaEvent_t ev = static_cast<cudaEvent_t>(t_trail.events[t_trail.next++]);
        if (ev) cudaEventRecord(ev, stream);
    }
}

namespace {

// A kernel that waits on a barrier nobody arrives at, bounded by limit_ns: exercises the timeout path.
__global__ void selftest_timeout_kernel(uint64_t limit_ns, int* status) {
    __shared__ uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        abort_flag = 0;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        const uint64_t t0 = globaltimer();
        bool ok = false;
        for (uint32_t i = 0; i < kWaitIterCap; ++i) {
            if (mbar_try_wait(&bar, 0)) { ok = true; break; }
            if ((i & 31u) == 31u && globaltimer() - t0 > limit_ns) break;
        }
        if (!ok) atomicExch(status, (int)ENTMAX_ERR_TIMEOUT);
        mbar_arrive(&bar);  // complete the phase so the barrier is left in a clean state
    }
}

int* status_ptr() {
    static int* cache[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!cache[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
        cache[dev] = static_cast<int*>(p);
    }
    return cache[dev];
}

inline size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct Dims {
    int B, H, n, d, mb, nqb, nkb, nw, nwq, bins, ntiles;
    entmax_dtype dt;
};

entmax_status check_dims(int B, int H, int n, int d, entmax_dtype dt, const entmax_opts* o, Dims* out) {
    if (B < 1 || H < 1 || n < 1 || d < 1) return ENTMAX_ERR_INVALID;
    if ((long long)B * H > (1ll << 30) || (long long)n > (1ll << 30)) return ENTMAX_ERR_INVALID;
    // the kernels' grids are (B*H, tiles of 128 rows); a grid's y extent is at most 65535
    if ((long long)n > 65535ll * kTileRows) return ENTMAX_ERR_UNSUPPORTED;
    if (dt != ENTMAX_BF16 && dt != ENTMAX_FP32) return ENTMAX_ERR_INVALID;
    if (d != 64 && d != 128) return ENTMAX_ERR_UNSUPPORTED;
    const int mb = (o && o->mask_block) ? o->mask_block : 64;
    if (mb != 32 && mb != 64) return ENTMAX_ERR_UNSUPPORTED;
    if (dt == ENTMAX_BF16 && mb != 64) return ENTMAX_ERR_UNSUPPORTED;
    const int bins = (o && o->hist_bins) ? o->hist_bins : 256;
    if (bins != 64 && bins != 128 && bins != 256 && bins != 512) return ENTMAX_ERR_UNSUPPORTED;
    if (o && (o->init_mode < 0 || o->init_mode > 1)) return ENTMAX_ERR_INVALID;
    if (o && o->scale != 0.0f && !(o->scale > 0.0f && isfinite(o->scale))) return ENTMAX_ERR_INVALID;
    if (o && (o->num_events < 0 || (o->num_events > 0 && !o->events))) return ENTMAX_ERR_INVALID;
    Dims D;
    D.B = B; D.H = H; D.n = n; D.d = d; D.mb = mb; D.bins = bins; D.dt = dt;
    D.nqb = (n + mb - 1) / mb;
    D.nkb = (n + mb - 1) / mb;
    D.nw = (D.nkb + 31) / 32;
    D.nwq = (D.nqb + 31) / 32;
    D.ntiles = (n + kTileRows - 1) / kTileRows;
    *out = D;
    return ENTMAX_OK;
}

// Workspace, in two parts.
//   saved   - what the backward needs from the forward: sum u ([BH][n]), the transposed mask and, for the
//             bf16 and fp32 kernels (not the fp16 family, whose dQ kernel forms delta itself), U V (fp32
//             [BH][n][d]);
//   scratch - per call: delta and the row statistic padded to whole 64-row blocks ([BH][ceil(n/64)*64]) for
//             the backward, the range words, and (bf16 inputs with d = 64, the only shape an fp16 kernel
//             serves) the fp16 operand copies of Q, K, V, dO (f16.cu).
// With one buffer (opts->scratch NULL) the scratch part follows the saved part, and a backward reuses the
// fp16 copies its forward left there; with a separate scratch buffer the backward makes its own copies.
struct Workspace {
    float* obar;
    float* sum_u;
    uint32_t* maskT;
    float* delta_pad;
    float* stat_pad;
    uint32_t* maxbits;  // [8]: max |x| of Q, K, V, dO, as float bits
    void* Qh;           // fp16 copies [BH][n][d] (f16.cu)
    void* Kh;
    void* Vh;
    void* dOh;
    size_t saved_bytes;
    size_t scratch_bytes;
    bool separate;      // scratch in its own buffer
};

Workspace layout(const Dims& D, void* base, void* scratch, bool with_obar) {
    const size_t rows = (size_t)D.B * D.H * D.n;
    const size_t rows_pad = (size_t)D.B * D.H * (size_t)((D.n + 63) / 64) * 64;
    Workspace w;
    char* p = static_cast<char*>(base);
    size_t off = 0;
    w.obar = nullptr;
    if (with_obar) {
        w.obar = reinterpret_cast<float*>(p + off);
        off = align256(off + rows * D.d * sizeof(float));
    }
    w.sum_u = reinterpret_cast<float*>(p + off);
    off = align256(off + rows * sizeof(float));
    w.maskT = reinterpret_cast<uint32_t*>(p + off);
    off = align256(off + (size_t)D.B * D.H * D.nkb * D.nwq * sizeof(uint32_t));
    w.saved_bytes = off;
    w.separate = scratch != nullptr;
    char* q = scratch ? static_cast<char*>(scratch) : p + off;
    size_t so = 0;
    w.delta_pad = reinterpret_cast<float*>(q + so);
    so = align256(so + rows_pad * sizeof(float));
    w.stat_pad = reinterpret_cast<float*>(q + so);
    so = align256(so + rows_pad * sizeof(float));
    w.maxbits = reinterpret_cast<uint32_t*>(q + so);
    so = align256(so + 8 * sizeof(uint32_t));
    void** h16[4] = {&w.Qh, &w.Kh, &w.Vh, &w.dOh};
    const bool with_h16 = D.dt == ENTMAX_BF16 && D.d == 64;
    for (int i = 0; i < 4; ++i) {
        *h16[i] = with_h16 ? q + so : nullptr;
        if (with_h16) so = align256(so + rows * D.d * 2);
    }
    w.scratch_bytes = so;
    return w;
}

entmax_status check_workspace(const Dims& D, const entmax_opts* o, Workspace* w, bool with_obar) {
    if (!o || !o->workspace) return ENTMAX_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(o->workspace) & 255u) != 0) return ENTMAX_ERR_ALIGN;
    if (o->scratch && (reinterpret_cast<uintptr_t>(o->scratch) & 255u) != 0) return ENTMAX_ERR_ALIGN;
    *w = layout(D, o->workspace, o->scratch, with_obar);
    if (o->scratch) {
        if (o->workspace_bytes < w->saved_bytes || o->scratch_bytes < w->scratch_bytes) return ENTMAX_ERR_WORKSPACE;
    } else if (o->workspace_bytes < w->saved_bytes + w->scratch_bytes) {
        return ENTMAX_ERR_WORKSPACE;
    }
    return ENTMAX_OK;
}

inline entmax_status from_cuda(cudaError_t e) { return e == cudaSuccess ? ENTMAX_OK : ENTMAX_ERR_CUDA; }

bool use_f16_path(int d, float alpha, int nw, int bins);

// U V is part of the saved workspace unless the fp16 family serves the call (bf16, d = 64, alpha <= 2).
// alpha <= 1 (unknown, for sizing) keeps it.
inline bool needs_obar(const Dims& D, float alpha, entmax_dtype dt) {
    return !(dt == ENTMAX_BF16 && alpha > 1.0f && use_f16_path(D.d, alpha, D.nw, D.bins));
}

int num_sms() {
    static int cache[64] = {0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
    if (!cache[dev]) {
        int v = 0;
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v < 1) v = 148;
        cache[dev] = v;
    }
    return cache[dev];
}

// The fp16 forward (fwd_h.cu) serves bf16 inputs with d = 64 and alpha <= 2 (p and u in [0, 1]), as long as
// its shared memory (which grows with the number of mask words per row and with the histogram size) fits;
// the backward follows the forward's choice (it reads the forward's fp16 copies).
constexpr size_t kMaxDynSmem = 232448;
bool use_f16_path(int d, float alpha, int nw, int bins) {
    return d == 64 && alpha <= 2.0f && fwd_h_smem_bytes(nw, bins) <= kMaxDynSmem;
}

}  // namespace
}  // namespace eattn

using namespace eattn;

#define EATTN_API __attribute__((visibility("default")))

extern "C" {

EATTN_API int entmax_attn_version(void) { return 3; }

EATTN_API const char* entmax_status_str(entmax_status s) {
    switch (s) {
        case ENTMAX_OK: return "ok";
        case ENTMAX_ERR_INVALID: return "invalid argument";
        case ENTMAX_ERR_UNSUPPORTED: return "unsupported configuration";
        case ENTMAX_ERR_ALIGN: return "pointer not aligned (16 bytes for tensors, 256 for the workspace)";
        case ENTMAX_ERR_CUDA: return "CUDA error";
        case ENTMAX_ERR_TIMEOUT: return "device-side wait timed out";
        case ENTMAX_ERR_WORKSPACE: return "workspace missing or too small";
    }
    return "unknown status";
}

EATTN_API size_t entmax_attn_workspace_size(int B, int H, int n, int d, entmax_dtype dt, const entmax_opts* opts) {
    Dims D;
    if (check_dims(B, H, n, d, dt, opts, &D) != ENTMAX_OK) return 0;
    const Workspace w = layout(D, nullptr, nullptr, needs_obar(D, opts ? opts->alpha : 0.0f, dt));
    return w.saved_bytes + w.scratch_bytes;
}

EATTN_API size_t entmax_attn_saved_size(int B, int H, int n, int d, entmax_dtype dt, const entmax_opts* opts) {
    Dims D;
    if (check_dims(B, H, n, d, dt, opts, &D) != ENTMAX_OK) return 0;
    return layout(D, nullptr, nullptr, needs_obar(D, opts ? opts->alpha : 0.0f, dt)).saved_bytes;
}

EATTN_API size_t entmax_attn_scratch_size(int B, int H, int n, int d, entmax_dtype dt, const entmax_opts* opts) {
    Dims D;
    if (check_dims(B, H, n, d, dt, opts, &D) != ENTMAX_OK) return 0;
    return layout(D, nullptr, nullptr, false).scratch_bytes;
}

EATTN_API size_t softmax_attn_workspace_size(int B, int H, int n, int d, entmax_dtype dt, const entmax_opts* opts) {
    Dims D;
    if (check_dims(B, H, n, d, dt, opts, &D) != ENTMAX_OK) return 0;
    const Workspace w = layout(D, nullptr, nullptr, false);
    return w.saved_bytes + w.scratch_bytes;
}

EATTN_API entmax_status entmax_attn_fwd(const void* Q, const void* K, const void* V, void* O, float* tau,
                              uint32_t* block_mask, int B, int H, int n, int d, float alpha, int causal,
                              entmax_dtype dt, const entmax_opts* opts, void* stream) {
    if (!Q || !K || !V || !O || !tau || !block_mask) return ENTMAX_ERR_INVALID;
    if (!(alpha > 1.0f) || !isfinite(alpha) || (causal != 0 && causal != 1)) return ENTMAX_ERR_INVALID;
    Dims D;
    entmax_status st = check_dims(B, H, n, d, dt, opts, &D);
    if (st != ENTMAX_OK) return st;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return ENTMAX_ERR_ALIGN;
    Workspace ws;
    if ((st = check_workspace(D, opts, &ws, needs_obar(D, alpha, dt))) != ENTMAX_OK) return st;
    int* status = status_ptr();
    if (!status) return ENTMAX_ERR_CUDA;

    FwdArgs a;
    memset(&a, 0, sizeof(a));
    a.Q = Q; a.K = K; a.V = V; a.O = O; a.tau = tau; a.mask = block_mask;
    a.obar = ws.obar; a.sum_u = ws.sum_u;
    a.tau_hist = opts->tau_hist; a.steps = opts->steps; a.stats = opts->stats; a.status = status;
    a.B = B; a.H = H; a.n = n; a.d = d;
    a.nqb = D.nqb; a.nkb = D.nkb; a.nw = D.nw; a.mb = D.mb; a.causal = causal; a.ntiles = D.ntiles;
    const float scale = opts->scale != 0.0f ? opts->scale : 1.0f / sqrtf((float)d);
    a.sp = make_solve_params(alpha, scale, D.bins, opts->init_mode);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    // 512 bins fit only the fp16 forward's shared-memory plan
    if (D.bins > 256 && !(dt == ENTMAX_BF16 && use_f16_path(d, alpha, D.nw, D.bins))) return ENTMAX_ERR_UNSUPPORTED;
    TrailScope trail(opts, s);
    cudaError_t e;
    if (dt == ENTMAX_FP32) {
        e = launch_fwd_simt(a, true, s);
    } else if (use_f16_path(d, alpha, D.nw, D.bins)) {
        F16Job job;
        memset(&job, 0, sizeof(job));
        job.src[0] = Q; job.src[1] = K; job.src[2] = V;
        job.dst[0] = ws.Qh; job.dst[1] = ws.Kh; job.dst[2] = ws.Vh;
        job.maxbits = ws.maxbits;
        job.n16 = (size_t)B * H * n * d / 8;
        job.count = 3;
        a.Qh = ws.Qh; a.Kh = ws.Kh; a.Vh = ws.Vh; a.maxbits = ws.maxbits;
        e = launch_to_f16(job, num_sms(), s);
        if (e == cudaSuccess) e = launch_fwd_h(a, s);
        if (e == cudaSuccess) e = launch_mask_transpose(block_mask, ws.maskT, B * H, D.nqb, D.nkb, D.nw, D.nwq, s);
    } else {
        e = launch_fwd_tc(a, s);
        if (e == cudaSuccess) e = launch_mask_transpose(block_mask, ws.maskT, B * H, D.nqb, D.nkb, D.nw, D.nwq, s);
    }
    return from_cuda(e);
}

EATTN_API entmax_status entmax_attn_check(void* stream) {
    cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return ENTMAX_ERR_CUDA;
    int* p = status_ptr();
    if (!p) return ENTMAX_ERR_CUDA;
    int v = 0;
    if (cudaMemcpy(&v, p, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return ENTMAX_ERR_CUDA;
    if (v != 0) {
        const int zero = 0;
        if (cudaMemcpy(p, &zero, sizeof(int), cudaMemcpyHostToDevice) != cudaSuccess) return ENTMAX_ERR_CUDA;
    }
    return static_cast<entmax_status>(v);
}

EATTN_API entmax_status entmax_attn_selftest_timeout(int limit_us, void* stream) {
    if (limit_us < 1 || limit_us > 2000000) return ENTMAX_ERR_INVALID;
    int* status = status_ptr();
    if (!status) return ENTMAX_ERR_CUDA;
    selftest_timeout_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>((uint64_t)limit_us * 1000ull, status);
    return from_cuda(cudaGetLastError());
}

}  // extern "C"


namespace {

entmax_status bwd_common(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                         const float* rowstat, const uint32_t* block_mask, void* dQ, void* dK, void* dV, int B,
                         int H, int n, int d, float alpha, int causal, entmax_dtype dt, const entmax_opts* opts,
                         void* stream, bool softmax) {
    if (!Q || !K || !V || !O || !dO || !rowstat || !dQ || !dK || !dV) return ENTMAX_ERR_INVALID;
    if (!softmax && !block_mask) return ENTMAX_ERR_INVALID;
    if (!softmax && (!(alpha > 1.0f) || !isfinite(alpha))) return ENTMAX_ERR_INVALID;
    if (causal != 0 && causal != 1) return ENTMAX_ERR_INVALID;
    Dims D;
    entmax_status st = check_dims(B, H, n, d, dt, opts, &D);
    if (st != ENTMAX_OK) return st;
    if (dt != ENTMAX_BF16) return ENTMAX_ERR_UNSUPPORTED;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O) || !aligned16(dO) || !aligned16(dQ) ||
        !aligned16(dK) || !aligned16(dV))
        return ENTMAX_ERR_ALIGN;
    Workspace ws;
    if ((st = check_workspace(D, opts, &ws, !softmax && needs_obar(D, alpha, dt))) != ENTMAX_OK) return st;
    int* status = status_ptr();
    if (!status) return ENTMAX_ERR_CUDA;
    const float scale = opts->scale != 0.0f ? opts->scale : 1.0f / sqrtf((float)d);
    BwdArgs a;
    memset(&a, 0, sizeof(a));
    a.Q = Q; a.K = K; a.V = V; a.O = O; a.dO = dO; a.rowstat = rowstat;
    a.mask = softmax ? nullptr : block_mask;
    a.maskT = softmax ? nullptr : ws.maskT;
    a.obar = ws.obar; a.sum_u = ws.sum_u;
    a.dQ = dQ; a.dK = dK; a.dV = dV; a.status = status;
    a.B = B; a.H = H; a.n = n; a.d = d;
    a.nqb = D.nqb; a.nkb = D.nkb; a.nw = D.nw; a.nwq = D.nwq;
    a.causal = causal; a.softmax = softmax ? 1 : 0; a.scale = scale;
    if (softmax) {
        a.cz = scale * 1.4426950408889634f;
        a.k = 1.0f;
        a.kind = 0;
    } else {
        const SolveParams sp = make_solve_params(alpha, scale, D.bins, 0);
        a.cz = sp.cz;
        a.k = sp.k;
        a.kind = alpha == 1.5f ? kAlpha15 : (alpha == 2.0f ? kAlpha2 : kGeneric);
    }
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TrailScope trail(opts, s);
    if (softmax && d == 64) {
        // dense baseline on the fp16 backward: it makes its own copies of Q, K, V and dO
        F16Job job;
        memset(&job, 0, sizeof(job));
        job.src[0] = Q; job.src[1] = K; job.src[2] = V; job.src[3] = dO;
        job.dst[0] = ws.Qh; job.dst[1] = ws.Kh; job.dst[2] = ws.Vh; job.dst[3] = ws.dOh;
        job.maxbits = ws.maxbits;
        job.n16 = (size_t)B * H * n * d / 8;
        job.count = 4;
        a.Qh = ws.Qh; a.Kh = ws.Kh; a.Vh = ws.Vh; a.dOh = ws.dOh; a.maxbits = ws.maxbits;
        cudaError_t e = launch_to_f16(job, num_sms(), s);
        if (e == cudaSuccess) e = launch_bwd_h(a, ws.delta_pad, ws.stat_pad, s);
        return from_cuda(e);
    }
    if (!softmax && use_f16_path(d, alpha, D.nw, D.bins)) {
        // fp16 path: with one workspace buffer the forward left fp16 copies of Q, K, V and their range
        // exponents in it and only dO is converted here; with a separate scratch buffer all four are
        F16Job job;
        memset(&job, 0, sizeof(job));
        if (ws.separate) {
            job.src[0] = Q; job.src[1] = K; job.src[2] = V; job.src[3] = dO;
            job.dst[0] = ws.Qh; job.dst[1] = ws.Kh; job.dst[2] = ws.Vh; job.dst[3] = ws.dOh;
            job.maxbits = ws.maxbits;
            job.count = 4;
        } else {
            job.src[0] = dO;
            job.dst[0] = ws.dOh;
            job.maxbits = ws.maxbits + 3;
            job.count = 1;
        }
        job.n16 = (size_t)B * H * n * d / 8;
        a.Qh = ws.Qh; a.Kh = ws.Kh; a.Vh = ws.Vh; a.dOh = ws.dOh; a.maxbits = ws.maxbits;
        cudaError_t e = launch_to_f16(job, num_sms(), s);
        if (e == cudaSuccess) e = launch_bwd_h(a, ws.delta_pad, ws.stat_pad, s);
        return from_cuda(e);
    }
    return from_cuda(launch_bwd(a, ws.delta_pad, ws.stat_pad, s));
}

}  // namespace

extern "C" {

EATTN_API entmax_status entmax_attn_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                                        const float* tau, const uint32_t* block_mask, void* dQ, void* dK, void* dV,
                                        int B, int H, int n, int d, float alpha, int causal, entmax_dtype dt,
                                        const entmax_opts* opts, void* stream) {
    return bwd_common(Q, K, V, O, dO, tau, block_mask, dQ, dK, dV, B, H, n, d, alpha, causal, dt, opts, stream,
                      false);
}

EATTN_API entmax_status softmax_attn_fwd(const void* Q, const void* K, const void* V, void* O, float* lse, int B,
                                         int H, int n, int d, int causal, entmax_dtype dt, const entmax_opts* opts,
                                         void* stream) {
    if (!Q || !K || !V || !O || !lse) return ENTMAX_ERR_INVALID;
    if (causal != 0 && causal != 1) return ENTMAX_ERR_INVALID;
    Dims D;
    entmax_status st = check_dims(B, H, n, d, dt, opts, &D);
    if (st != ENTMAX_OK) return st;
    if (dt != ENTMAX_BF16) return ENTMAX_ERR_UNSUPPORTED;
    if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O)) return ENTMAX_ERR_ALIGN;
    int* status = status_ptr();
    if (!status) return ENTMAX_ERR_CUDA;
    SoftmaxFwdArgs a;
    memset(&a, 0, sizeof(a));
    a.Q = Q; a.K = K; a.V = V; a.O = O; a.lse = lse; a.status = status;
    a.B = B; a.H = H; a.n = n; a.d = d; a.causal = causal; a.ntiles = D.ntiles;
    a.scale = (opts && opts->scale != 0.0f) ? opts->scale : 1.0f / sqrtf((float)d);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    TrailScope trail(opts, s);
    Workspace ws;
    if (d == 64 && opts && opts->workspace && check_workspace(D, opts, &ws, false) == ENTMAX_OK) {
        // fp16 path: copies of Q, K, V in the workspace
        F16Job job;
        memset(&job, 0, sizeof(job));
        job.src[0] = Q; job.src[1] = K; job.src[2] = V;
        job.dst[0] = ws.Qh; job.dst[1] = ws.Kh; job.dst[2] = ws.Vh;
        job.maxbits = ws.maxbits;
        job.n16 = (size_t)B * H * n * d / 8;
        job.count = 3;
        a.Qh = ws.Qh; a.Kh = ws.Kh; a.Vh = ws.Vh; a.maxbits = ws.maxbits;
        cudaError_t e = launch_to_f16(job, num_sms(), s);
        if (e == cudaSuccess) e = launch_softmax_fwd_h(a, s);
        return from_cuda(e);
    }
    return from_cuda(launch_softmax_fwd(a, s));
}

EATTN_API entmax_status softmax_attn_bwd(const void* Q, const void* K, const void* V, const void* O, const void* dO,
                                         const float* lse, void* dQ, void* dK, void* dV, int B, int H, int n, int d,
                                         int causal, entmax_dtype dt, const entmax_opts* opts, void* stream) {
    return bwd_common(Q, K, V, O, dO, lse, nullptr, dQ, dK, dV, B, H, n, d, 2.0f, causal, dt, opts, stream, true);
}

}  // extern "C"

// ---------------------------------------------------------------------------------------------
// Forward without caller-provided workspace (no allocation at all).
//
// Some callers cannot allocate device memory: code that runs while a host framework owns the whole
// device pool and exposes no allocator, or that must not call cudaMalloc on its path (it can
// synchronise the device, and it is not allowed while a stream is being captured). For them the
// forward can use a fixed scratch area that lives in the library image: a file-scope device array of
// kStaticScratchBytes, which every GPU that loads the library keeps until the process exits. Host code
// cannot use the array's name as a device address, so its address is looked up once per device.
// ---------------------------------------------------------------------------------------------
namespace eattn {
namespace {

constexpr size_t kStaticScratchBytes = (size_t)32 << 20;  // 32 MiB
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// Device address of the scratch array on the current device (looked up on the first call per device,
// with that device current). Returns nullptr if the lookup fails.
void* static_scratch_ptr() {
    static void* cache[64] = {nullptr};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!cache[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess || p == nullptr) return nullptr;
        cache[dev] = p;
    }
    return cache[dev];
}

}  // namespace
}  // namespace eattn

extern "C" {

EATTN_API entmax_status entmax_attn_fwd_noalloc(const void* Q, const void* K, const void* V, void* O, float* tau,
                                                uint32_t* block_mask, int B, int H, int n, int d, float alpha,
                                                int causal, entmax_dtype dt, const entmax_opts* opts, void* stream) {
    entmax_opts o;
    memset(&o, 0, sizeof(o));
    if (opts) o = *opts;
    o.scratch = nullptr;
    o.scratch_bytes = 0;
    const size_t need = entmax_attn_workspace_size(B, H, n, d, dt, &o);
    if (need == 0) {
        // let the regular checks name the problem (invalid or unsupported sizes)
        o.workspace = nullptr;
        o.workspace_bytes = 0;
        Dims D;
        const entmax_status st = check_dims(B, H, n, d, dt, &o, &D);
        return st != ENTMAX_OK ? st : ENTMAX_ERR_INVALID;
    }
    if (need > kStaticScratchBytes) return ENTMAX_ERR_WORKSPACE;
    void* scratch = static_scratch_ptr();
    if (!scratch) return ENTMAX_ERR_CUDA;
    o.workspace = scratch;
    o.workspace_bytes = kStaticScratchBytes;
    o.scratch = nullptr;
    o.scratch_bytes = 0;
    return entmax_attn_fwd(Q, K, V, O, tau, block_mask, B, H, n, d, alpha, causal, dt, &o, stream);
}

}  // extern "C"
