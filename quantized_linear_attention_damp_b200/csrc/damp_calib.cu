// damp_calib.cu -- offline calibration of the FP16 key rows: per-row INT8
// quantization-error energy and decay retention of an FP32 state pool
// (accumulate), scores and top-k selection (select, select_budget).
//
// "DAMP: Decay-Aware Mixed-Precision Recurrent-State Quantization" (both
// abstracts) selects the high-risk key channels offline from the
// quantization-error energy and the decay-based error retention of each
// channel, under a fixed storage budget.  The formulas are readings stated in
// damp.h.
//
// Accumulate: one warp owns one (head, key row) total and walks the batch in
// order, so the sums do not depend on scheduling.  Four batch entries are
// loaded before any is reduced to keep several row reads in flight per warp.
#include <cuda_runtime.h>

#include <mutex>

#include "damp.h"
#include "damp_device.cuh"
#include "damp_internal.h"

namespace damp {
namespace {

constexpr int kCalRows = 8;      // key rows (warps) per CTA
constexpr int kCalUnroll = 4;    // batch entries loaded per round

// Quantization error energy of the elements a lane holds, for a row with
// scale s / inverse inv (the decode step's quantizer): code = RNE(x*inv) by
// one fma against 1.5*2^23, dequantized as fl(code*s), error squared in
// double (x - dq is exact in double).
__device__ __forceinline__ double lane_error(float x, float s, float inv) {
    const float c = __fsub_rn(__fmaf_rn(x, inv, 12582912.0f), 12582912.0f);
    const float dq = __fmul_rn(c, s);
    const double df = __dsub_rn((double)x, (double)dq);
    return __dmul_rn(df, df);
}

__device__ __forceinline__ double warp_sum(double v) {
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) v = __dadd_rn(v, __shfl_xor_sync(0xffffffffu, v, off));
    return v;
}

// Warp (h, i) owns the totals of key row i of head h; lane l holds columns
// l + 32t (t < EPL) of the row, zero past d_v (a zero adds no error).
template <int EPL>
__global__ void __launch_bounds__(kCalRows * 32)
    calib_accumulate_kernel(CalibArgs a) {
    const int lane = threadIdx.x & 31;
    const int h = blockIdx.x;
    const int d_k = a.d_k, d_v = a.d_v;
    const int i = blockIdx.y * kCalRows + (threadIdx.x >> 5);
    if (i >= d_k) return;
    const size_t hi = (size_t)h * d_k + i;
    double* energy = a.acc;
    double* retention = a.acc + (size_t)a.H * d_k;
    double* count = a.acc + 2 * (size_t)a.H * d_k;
    double e_acc = energy[hi], r_acc = retention[hi];
    int cnt = 0;

    for (int b0 = 0; b0 < a.n; b0 += kCalUnroll) {
        int slot[kCalUnroll];
        float x[kCalUnroll][EPL];
#pragma unroll
        for (int u = 0; u < kCalUnroll; ++u) {
            const int b = b0 + u;
            slot[u] = b < a.n ? __ldg(a.slot_idx + b) : -1;
            const bool ok = slot[u] >= 0 && slot[u] < a.n_slots;
            const float* row = a.state + ((size_t)(ok ? slot[u] : 0) * a.H + h) * d_k * d_v +
                               (size_t)i * d_v;
#pragma unroll
            for (int t = 0; t < EPL; ++t) {
                const int j = lane + 32 * t;
                x[u][t] = (ok && j < d_v) ? __ldg(row + j) : 0.0f;
            }
        }
#pragma unroll
        for (int u = 0; u < kCalUnroll; ++u) {
            const int b = b0 + u;
            if (b >= a.n || slot[u] < 0) continue;   // warp-uniform
            if (slot[u] >= a.n_slots) {
                if (i == 0 && lane == 0) atomicOr(a.status, DAMP_EFLAG_SLOT_RANGE);
                continue;
            }
            float m = 0.0f;
#pragma unroll
            for (int t = 0; t < EPL; ++t) m = fmaxf(m, fabsf(x[u][t]));
            m = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m)));
            float s, inv;
            row_scale(m, s, inv);
            double e = 0.0;
#pragma unroll
            for (int t = 0; t < EPL; ++t) e = __dadd_rn(e, lane_error(x[u][t], s, inv));
            e = warp_sum(e);
            const float al = a.gate == DAMP_GATE_VECTOR
                                 ? __ldg(a.alpha + ((size_t)b * a.H + h) * d_k + i)
                                 : __ldg(a.alpha + (size_t)b * a.H + h);
            e_acc = __dadd_rn(e_acc, e);
            r_acc = __dadd_rn(r_acc, __dmul_rn((double)al, (double)al));
            ++cnt;
        }
    }
    if (lane == 0) {
        energy[hi] = e_acc;
        retention[hi] = r_acc;
        if (i == 0) count[h] = __dadd_rn(count[h], (double)cnt);
    }
}

__device__ __forceinline__ double calib_score(const double* acc, int H, int D, int h, int i) {
    const double c = acc[2 * (size_t)H * D + h];
    if (c <= 0.0) return 0.0;
    const double E = __ddiv_rn(acc[(size_t)h * D + i], c);
    double keep = __dsub_rn(1.0, __ddiv_rn(acc[(size_t)H * D + (size_t)h * D + i], c));
    constexpr double fl = 1.0 / 1073741824.0;   // 2^-30
    if (keep < fl) keep = fl;
    return __ddiv_rn(E, keep);
}

// One CTA per head, one thread per key row: rank by counting (ties to the
// lower row), then the selected rows' positions by a prefix count.
__global__ void __launch_bounds__(kMaxDim)
    calib_select_kernel(const double* acc, int H, int D, int hp, double* score,
                        uint16_t* idx) {
    __shared__ double sc[kMaxDim];
    __shared__ int sel[kMaxDim];
    const int h = blockIdx.x, i = threadIdx.x;
    const double s = i < D ? calib_score(acc, H, D, h, i) : 0.0;
    sc[i] = s;
    __syncthreads();
    int take = 0;
    if (i < D) {
        int rank = 0;
        for (int j = 0; j < D; ++j) rank += (sc[j] > s) || (sc[j] == s && j < i);
        take = rank < hp;
        if (score) score[(size_t)h * D + i] = s;
    }
    sel[i] = take;
    __syncthreads();
    if (take) {
        int pos = 0;
        for (int j = 0; j < i; ++j) pos += sel[j];
        idx[(size_t)h * hp + pos] = (uint16_t)i;
    }
}

__global__ void calib_score_kernel(const double* acc, int H, int D, double* score) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e < H * D) score[e] = calib_score(acc, H, D, e / D, e % D);
}

// Rank of every (head, row) among all H*D scores, by counting over shared
// memory tiles; ties go to the lower flat index (lower head, then row).
__global__ void __launch_bounds__(256)
    calib_budget_kernel(const double* score, int total, int budget, uint8_t* is_fp16) {
    __shared__ double tile[256];
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    const double s = e < total ? score[e] : 0.0;
    int rank = 0;
    for (int t0 = 0; t0 < total; t0 += 256) {
        const int f = t0 + threadIdx.x;
        tile[threadIdx.x] = f < total ? score[f] : 0.0;
        __syncthreads();
        const int lim = min(256, total - t0);
        for (int j = 0; j < lim; ++j) {
            const double o = tile[j];
            rank += (o > s) || (o == s && t0 + j < e);
        }
        __syncthreads();
    }
    if (e < total) is_fp16[e] = rank < budget ? 1 : 0;
}

__global__ void calib_count_kernel(const uint8_t* is_fp16, int D, int32_t* hp) {
    __shared__ int c;
    if (threadIdx.x == 0) c = 0;
    __syncthreads();
    int mine = 0;
    for (int i = threadIdx.x; i < D; i += blockDim.x) mine += is_fp16[(size_t)blockIdx.x * D + i];
    atomicAdd(&c, mine);
    __syncthreads();
    if (threadIdx.x == 0) hp[blockIdx.x] = c;
}

}  // namespace

cudaError_t launch_calib_accumulate(const CalibArgs& a, cudaStream_t stream) {
    const dim3 grid(a.H, (a.d_k + kCalRows - 1) / kCalRows);
    switch ((a.d_v + 31) / 32) {
        case 1: calib_accumulate_kernel<1><<<grid, kCalRows * 32, 0, stream>>>(a); break;
        case 2: calib_accumulate_kernel<2><<<grid, kCalRows * 32, 0, stream>>>(a); break;
        case 3: calib_accumulate_kernel<3><<<grid, kCalRows * 32, 0, stream>>>(a); break;
        case 4: calib_accumulate_kernel<4><<<grid, kCalRows * 32, 0, stream>>>(a); break;
        case 5: calib_accumulate_kernel<5><<<grid, kCalRows * 32, 0, stream>>>(a); break;
        case 6: calib_accumulate_kernel<6><<<grid, kCalRows * 32, 0, stream>>>(a); break;
        case 7: calib_accumulate_kernel<7><<<grid, kCalRows * 32, 0, stream>>>(a); break;
        case 8: calib_accumulate_kernel<8><<<grid, kCalRows * 32, 0, stream>>>(a); break;
        default: return cudaErrorInvalidValue;
    }
    return cudaGetLastError();
}

cudaError_t launch_calib_select(const double* acc, int H, int d, int hp, double* score,
                                uint16_t* idx, cudaStream_t stream) {
    calib_select_kernel<<<H, kMaxDim, 0, stream>>>(acc, H, d, hp, score, idx);
    return cudaGetLastError();
}

cudaError_t launch_calib_select_budget(const double* acc, int H, int d, int budget,
                                       double* score, uint8_t* is_fp16, int32_t* hp,
                                       cudaStream_t stream) {
    const int total = H * d;
    calib_score_kernel<<<(total + 255) / 256, 256, 0, stream>>>(acc, H, d, score);
    calib_budget_kernel<<<(total + 255) / 256, 256, 0, stream>>>(score, total, budget, is_fp16);
    calib_count_kernel<<<H, 128, 0, stream>>>(is_fp16, d, hp);
    return cudaGetLastError();
}

}  // namespace damp

// ---------------------------------------------------------------------------
// Budget selection with library-owned scratch: the scores live in a static
// device array instead of a caller buffer, so the call allocates nothing.
// ---------------------------------------------------------------------------
namespace damp {
namespace {

constexpr int kStaticScores = DAMP_SELECT_BUDGET_STATIC_MAX;   // 128 KiB of doubles

// Every device that loads the library holds one copy until the process exits.
static __device__ __align__(256) double g_budget_scores[kStaticScores];

// Device address of g_budget_scores on each device, looked up once per device
// with that device current (in host code the symbol itself is only a host-side
// stand-in and must never reach a kernel).
constexpr int kMaxDevices = 64;
std::mutex g_scores_mu;
double* g_scores_addr[kMaxDevices] = {};

cudaError_t static_scores(double** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_scores_mu);
    if (!g_scores_addr[dev]) {
        void* p = nullptr;
        e = cudaGetSymbolAddress(&p, g_budget_scores);
        if (e != cudaSuccess) return e;
        g_scores_addr[dev] = static_cast<double*>(p);
    }
    *out = g_scores_addr[dev];
    return cudaSuccess;
}

}  // namespace
}  // namespace damp

extern "C" int damp_calib_select_budget_static(int H, int d_k, int budget, const double* acc,
                                               uint8_t* is_fp16, int32_t* hp_per_head,
                                               void* stream) {
    if (H <= 0 || d_k <= 0) return DAMP_ERR_INVALID_ARGUMENT;
    if (d_k < 16 || d_k > damp::kMaxDim || d_k % 16) return DAMP_ERR_UNSUPPORTED;
    if ((size_t)H * d_k > (size_t)damp::kStaticScores) return DAMP_ERR_UNSUPPORTED;
    if (budget < 0 || budget > H * d_k || !acc || !is_fp16 || !hp_per_head)
        return DAMP_ERR_INVALID_ARGUMENT;
    if ((reinterpret_cast<uintptr_t>(acc) & 7u) || (reinterpret_cast<uintptr_t>(hp_per_head) & 3u))
        return DAMP_ERR_MISALIGNED;
    double* scores = nullptr;
    if (damp::static_scores(&scores) != cudaSuccess) return DAMP_ERR_CUDA;
    const cudaError_t e = damp::launch_calib_select_budget(acc, H, d_k, budget, scores, is_fp16,
                                                           hp_per_head,
                                                           static_cast<cudaStream_t>(stream));
    return e == cudaSuccess ? DAMP_OK : DAMP_ERR_CUDA;
}

