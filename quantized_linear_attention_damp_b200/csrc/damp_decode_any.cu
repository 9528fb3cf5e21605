// damp_decode_any.cu -- decode step, pack and unpack for every state shape
// d_k x d_v (multiples of 16 up to 256, d_k != d_v allowed) and every format.
//
// The square shapes d in {16, 32, 64, 128} have faster kernels
// (damp_decode.cu, damp_decode_unit.cu, damp_codec.cu); these kernels serve
// every other shape.  Same arithmetic, same order of operations and the same
// stored bytes as those kernels and as the oracle ("STEPQuant ...", Appendix
// Table C2 steps 1, 2, 3, 6 on the DAMP row format).
//
// Decode: one CTA of 256 threads per unit (slot, head), working on the block
// in global memory (a block can be 256 KB, more than shared memory holds).
//   pass 1  thread j < d_v owns column j: it walks the key rows in order,
//           forms S'_ij = fl(alpha_i * S^_ij), adds the leaf fl(k_i S'_ij) to
//           the recursive pairwise sum u_j (the oracle's halving tree for
//           d_k rows: a stack and, per row, the number of merges that follow
//           it), and accumulates w_j = q^T S'_:j;
//   then    delta_j = fl(v_j - u_j), out_j = fma(c, delta_j, w_j) with
//           c = q^T (beta k);
//   pass 2  warp w takes key rows w, w + 8, ...: it recomputes S'_i: (the
//           same roundings), forms X_i: = fma(b_i, delta, S'_i:) and stores
//           the row in its format (FP32, FP16, or bytes with the row's new
//           scale).  Every read of pass 1 is done before pass 2 writes (one
//           CTA barrier), and a row is read and written by one warp only.
// Pack and unpack: one warp per (unit, key row).
#include <cuda_runtime.h>

#include <algorithm>

#include "damp.h"
#include "damp_device.cuh"

namespace damp {
namespace {

constexpr int kAnyThreads = 256;
constexpr int kAnyWarps = kAnyThreads / 32;
constexpr int kColsPerLane = kMaxDim / 32;   // columns a lane holds in pass 2

__device__ __forceinline__ float in_val(const void* base, size_t idx, bool bf16) {
    if (bf16)
        return __uint_as_float(static_cast<uint32_t>(static_cast<const uint16_t*>(base)[idx]) << 16);
    return static_cast<const float*>(base)[idx];
}

// Value of one E4M3 code (exact).
__device__ __forceinline__ float e4m3_value(uint8_t c) {
    uint32_t h;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"((unsigned short)c));
    return __half2float(__ushort_as_half((unsigned short)(h & 0xffffu)));
}

// E4M3 code of y (nearest, ties to even, saturating at 448).
__device__ __forceinline__ uint8_t e4m3_code(float y) {
    unsigned short p;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(p) : "f"(0.0f), "f"(y));
    return (uint8_t)(p & 0xffu);
}

// Element j of stored row i, before the decay: S^_ij.  codec: 0 FP32 state,
// 1 INT8 rows, 2 FP8 rows; e = the row's directory word; s = its scale.
__device__ __forceinline__ float load_shat(const uint8_t* blk, int codec, uint32_t e, float s,
                                           int i, int j, int d_v) {
    if (codec == 0) return reinterpret_cast<const float*>(blk)[(size_t)i * d_v + j];
    const uint8_t* row = blk + dir_row(e);
    if (e >> 31) return __half2float(*reinterpret_cast<const __half*>(row + f16_pos(j, d_v)));
    if (codec == 2) return __fmul_rn(e4m3_value(row[j]), s);
    return __fmul_rn((float)(int8_t)row[j], s);
}

// The aligned word of the block that holds element j of stored row i (any
// format: the word of an FP16 or byte row lies inside the row), and the
// element's value read from that word.  Splitting the two lets a thread put
// the loads of several rows in flight before it needs the first value.
__device__ __forceinline__ const uint32_t* shat_word(const uint8_t* blk, int codec, uint32_t e,
                                                     int i, int j, int d_v) {
    if (codec == 0) return reinterpret_cast<const uint32_t*>(blk) + (size_t)i * d_v + j;
    const uint32_t off = (e >> 31) ? f16_pos(j, d_v) : (uint32_t)j;
    return reinterpret_cast<const uint32_t*>(blk + dir_row(e) + (off & ~3u));
}
__device__ __forceinline__ float shat_from_word(uint32_t w, int codec, uint32_t e, float s, int j,
                                                int d_v) {
    if (codec == 0) return __uint_as_float(w);
    if (e >> 31)
        return __half2float(__ushort_as_half((unsigned short)(w >> ((f16_pos(j, d_v) & 2u) * 8u))));
    const uint8_t b = (uint8_t)(w >> (8u * ((uint32_t)j & 3u)));
    if (codec == 2) return __fmul_rn(e4m3_value(b), s);
    return __fmul_rn((float)(int8_t)b, s);
}

// Row operands of one unit, in shared memory.
struct AnyRows {
    float k[kMaxDim], q[kMaxDim], b[kMaxDim], al[kMaxDim], s[kMaxDim];
    uint32_t e[kMaxDim];
    uint8_t merges[kMaxDim];   // pairwise merges after leaf i
};

__global__ void __launch_bounds__(kAnyThreads) decode_any_kernel(const StepArgs a, int codec,
                                                                 int kda, int bf16) {
    __shared__ AnyRows R;
    __shared__ float s_delta[kMaxDim];
    __shared__ float s_c[kAnyWarps];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int d_k = a.d_k, d_v = a.d_v;
    const long long u = blockIdx.x;   // unit b*H + h
    const int b = (int)(u / a.H), h = (int)(u % a.H);
    float* out = a.out + (size_t)u * d_v;
    const int slot = __ldg(a.slot_idx + b);
    if (slot < 0 || slot >= a.n_slots) {
        for (int j = tid; j < d_v; j += kAnyThreads) out[j] = 0.f;
        if (slot >= a.n_slots && tid == 0) atomicOr(a.status, DAMP_EFLAG_SLOT_RANGE);
        return;
    }
    const uint4 hb = __ldg(a.heads + h);
    uint8_t* blk = a.blocks + (size_t)slot * a.slot_stride + hb.x;
    const float beta = __ldg(a.beta + u);
    const float alpha_g = kda ? 0.f : __ldg(a.alpha + u);

    // ---- per-row operands and the pairwise merge schedule of d_k leaves
    if (tid == 0) {
        for (int i = 0; i < d_k; ++i) R.merges[i] = 0;
        // internal node (lo, n) of the halving tree: its sum is formed right
        // after its last leaf lo + n - 1 (explicit stack of ranges)
        int st_lo[2 * 9], st_n[2 * 9], top = 0;
        st_lo[0] = 0;
        st_n[0] = d_k;
        top = 1;
        while (top > 0) {
            --top;
            const int lo = st_lo[top], n = st_n[top];
            if (n <= 1) continue;
            R.merges[lo + n - 1] += 1;
            const int hh = n / 2;
            st_lo[top] = lo + hh;
            st_n[top] = n - hh;
            ++top;
            st_lo[top] = lo;
            st_n[top] = hh;
            ++top;
        }
    }
    bool bad = false;
    for (int i = tid; i < d_k; i += kAnyThreads) {
        const float kr = in_val(a.k, (size_t)u * d_k + i, bf16);
        const float qr = in_val(a.q, (size_t)u * d_k + i, bf16);
        const float al = kda ? __ldg(a.alpha + (size_t)u * d_k + i) : alpha_g;
        const uint32_t e = codec ? __ldg(a.dir + (size_t)h * d_k + i) : 0u;
        R.k[i] = kr;
        R.q[i] = qr;
        R.b[i] = __fmul_rn(beta, kr);
        R.al[i] = al;
        R.e[i] = e;
        R.s[i] = (codec && !(e >> 31)) ? *reinterpret_cast<const float*>(blk + dir_scale(e)) : 1.0f;
        bad |= !(isfinite(kr) && isfinite(qr) && isfinite(al));
    }
    if (a.validate) {
        for (int j = tid; j < d_v; j += kAnyThreads)
            bad |= !isfinite(in_val(a.v, (size_t)u * d_v + j, bf16));
        bad |= !isfinite(beta) || (!kda && !isfinite(alpha_g));
        if (__syncthreads_or(bad)) {
            for (int j = tid; j < d_v; j += kAnyThreads) out[j] = 0.f;
            if (tid == 0) atomicOr(a.status, DAMP_EFLAG_NONFINITE);
            return;   // uniform: the block is neither read further nor written
        }
    } else {
        __syncthreads();
    }

    // c = q^T (beta k), any order
    {
        float cp = 0.f;
        for (int i = tid; i < d_k; i += kAnyThreads) cp = __fadd_rn(cp, __fmul_rn(R.q[i], R.b[i]));
#pragma unroll
        for (int off = 16; off >= 1; off >>= 1) cp += __shfl_xor_sync(0xffffffffu, cp, off);
        if (lane == 0) s_c[warp] = cp;
    }

    // ---- pass 1: column j
    float uj = 0.f, wj = 0.f;
    if (tid < d_v) {
        const int j = tid;
        float stk[10];
        int top = 0;
        // rows in batches of 8 (d_k is a multiple of 16): the batch's loads first
        for (int i0 = 0; i0 < d_k; i0 += 8) {
            uint32_t w[8];
#pragma unroll
            for (int t = 0; t < 8; ++t) w[t] = *shat_word(blk, codec, R.e[i0 + t], i0 + t, j, d_v);
#pragma unroll
            for (int t = 0; t < 8; ++t) {
                const int i = i0 + t;
                const float sp =
                    __fmul_rn(R.al[i], shat_from_word(w[t], codec, R.e[i], R.s[i], j, d_v));
                wj = __fmaf_rn(R.q[i], sp, wj);
                stk[top++] = __fmul_rn(R.k[i], sp);   // leaf fl(k_i S'_ij)
                for (int m = R.merges[i]; m > 0; --m) {
                    stk[top - 2] = __fadd_rn(stk[top - 2], stk[top - 1]);   // left + right
                    --top;
                }
            }
        }
        uj = stk[0];
    }
    __syncthreads();
    if (tid < d_v) {
        float c = 0.f;
#pragma unroll
        for (int w = 0; w < kAnyWarps; ++w) c += s_c[w];
        const float dj = __fsub_rn(in_val(a.v, (size_t)u * d_v + tid, bf16), uj);
        s_delta[tid] = dj;
        out[tid] = __fmaf_rn(c, dj, wj);
    }
    __syncthreads();

    // ---- pass 2: row i by warp, columns lane + 32t
    for (int i = warp; i < d_k; i += kAnyWarps) {
        const uint32_t e = R.e[i];
        float x[kColsPerLane];
        float m = 0.f;
#pragma unroll
        for (int t = 0; t < kColsPerLane; ++t) {
            const int j = lane + 32 * t;
            x[t] = 0.f;
            if (j < d_v) {
                const float sp = __fmul_rn(R.al[i], load_shat(blk, codec, e, R.s[i], i, j, d_v));
                x[t] = __fmaf_rn(R.b[i], s_delta[j], sp);
                m = fmaxf(m, fabsf(x[t]));
            }
        }
        if (codec == 0) {
#pragma unroll
            for (int t = 0; t < kColsPerLane; ++t) {
                const int j = lane + 32 * t;
                if (j < d_v) reinterpret_cast<float*>(blk)[(size_t)i * d_v + j] = x[t];
            }
            continue;
        }
        uint8_t* row = blk + dir_row(e);
        if (e >> 31) {
#pragma unroll
            for (int t = 0; t < kColsPerLane; ++t) {
                const int j = lane + 32 * t;
                if (j < d_v) *reinterpret_cast<__half*>(row + f16_pos(j, d_v)) = __float2half_rn(x[t]);
            }
            continue;
        }
        m = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m)));
        float scale, inv;
        if (codec == 2) row_scale<true>(m, scale, inv);
        else row_scale<false>(m, scale, inv);
#pragma unroll
        for (int t = 0; t < kColsPerLane; ++t) {
            const int j = lane + 32 * t;
            if (j >= d_v) continue;
            if (codec == 2) {
                row[j] = inv == 0.0f ? (uint8_t)0 : e4m3_code(__fmul_rn(x[t], inv));
            } else {
                // RNE of the exact x*inv: one fused multiply-add with 1.5*2^23
                row[j] = (uint8_t)(__float_as_uint(__fmaf_rn(x[t], inv, 12582912.0f)) & 0xffu);
            }
        }
        if (lane == 0) *reinterpret_cast<float*>(blk + dir_scale(e)) = scale;
    }
}

// Pack (FP32 states -> blocks) or unpack (blocks -> FP32 states): warp per
// (unit, key row), columns lane + 32t.
template <bool PACK>
__global__ void __launch_bounds__(kAnyThreads) codec_any_kernel(const CodecArgs a, int codec) {
    const int lane = threadIdx.x & 31;
    const long long row_id = (long long)blockIdx.x * kAnyWarps + (threadIdx.x >> 5);
    const long long n_rows = (long long)a.n * a.H * a.d_k;
    if (row_id >= n_rows) return;
    const int d_k = a.d_k, d_v = a.d_v;
    const long long u = row_id / d_k;
    const int i = (int)(row_id % d_k);
    const int b = (int)(u / a.H), h = (int)(u % a.H);
    float* st = a.state + ((size_t)u * d_k + i) * d_v;
    const int slot = __ldg(a.slot_idx + b);
    if (slot < 0 || slot >= a.n_slots) {
        if (!PACK)
            for (int j = lane; j < d_v; j += 32) st[j] = 0.f;
        if (slot >= a.n_slots && i == 0 && lane == 0) atomicOr(a.status, DAMP_EFLAG_SLOT_RANGE);
        return;
    }
    const uint4 hb = __ldg(a.heads + h);
    uint8_t* blk = a.blocks + (size_t)slot * a.slot_stride + hb.x;
    const uint32_t e = codec ? __ldg(a.dir + (size_t)h * d_k + i) : 0u;
    if constexpr (!PACK) {
        const float s = (codec && !(e >> 31)) ? *reinterpret_cast<const float*>(blk + dir_scale(e)) : 1.f;
        for (int j = lane; j < d_v; j += 32) st[j] = load_shat(blk, codec, e, s, i, j, d_v);
    } else {
        float x[kColsPerLane];
        float m = 0.f;
#pragma unroll
        for (int t = 0; t < kColsPerLane; ++t) {
            const int j = lane + 32 * t;
            x[t] = j < d_v ? __ldg(st + j) : 0.f;
            m = fmaxf(m, fabsf(x[t]));
        }
        if (codec == 0) {
#pragma unroll
            for (int t = 0; t < kColsPerLane; ++t) {
                const int j = lane + 32 * t;
                if (j < d_v) reinterpret_cast<float*>(blk)[(size_t)i * d_v + j] = x[t];
            }
            return;
        }
        uint8_t* row = blk + dir_row(e);
        if (e >> 31) {
#pragma unroll
            for (int t = 0; t < kColsPerLane; ++t) {
                const int j = lane + 32 * t;
                if (j < d_v) *reinterpret_cast<__half*>(row + f16_pos(j, d_v)) = __float2half_rn(x[t]);
            }
            return;
        }
        m = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m)));
        float scale, inv;
        if (codec == 2) row_scale<true>(m, scale, inv);
        else row_scale<false>(m, scale, inv);
#pragma unroll
        for (int t = 0; t < kColsPerLane; ++t) {
            const int j = lane + 32 * t;
            if (j >= d_v) continue;
            if (codec == 2) row[j] = inv == 0.0f ? (uint8_t)0 : e4m3_code(__fmul_rn(x[t], inv));
            else row[j] = (uint8_t)(__float_as_uint(__fmaf_rn(x[t], inv, 12582912.0f)) & 0xffu);
        }
        if (lane == 0) *reinterpret_cast<float*>(blk + dir_scale(e)) = scale;
    }
}

inline int codec_of_fmt(int format) {
    return format == DAMP_FMT_FP32 ? 0 : format == DAMP_FMT_FP8_ROW ? 2 : 1;
}

}  // namespace

cudaError_t launch_decode_any(const StepArgs& a, int in_dtype, int gate, cudaStream_t stream) {
    const long long units = (long long)a.n * a.H;
    if (units <= 0) return cudaSuccess;
    decode_any_kernel<<<(unsigned)units, kAnyThreads, 0, stream>>>(
        a, codec_of_fmt(a.format), gate == DAMP_GATE_VECTOR ? 1 : 0,
        in_dtype == DAMP_DTYPE_BF16 ? 1 : 0);
    return cudaGetLastError();
}

template <bool PACK>
static cudaError_t launch_codec_any(const CodecArgs& a, cudaStream_t stream) {
    const long long rows = (long long)a.n * a.H * a.d_k;
    if (rows <= 0) return cudaSuccess;
    const long long grid = (rows + kAnyWarps - 1) / kAnyWarps;
    codec_any_kernel<PACK><<<(unsigned)grid, kAnyThreads, 0, stream>>>(a, codec_of_fmt(a.format));
    return cudaGetLastError();
}

cudaError_t launch_pack_any(const CodecArgs& a, cudaStream_t stream) {
    return launch_codec_any<true>(a, stream);
}
cudaError_t launch_unpack_any(const CodecArgs& a, cudaStream_t stream) {
    return launch_codec_any<false>(a, stream);
}

}  // namespace damp
