// damp_device.cuh -- device helpers of libdamp: PTX wrappers for the bulk-copy
// pipeline and the per-thread tile codec (dequantize / requantize) shared by
// the decode-step and pack/unpack kernels.
//
// Arithmetic contract (every FP32 operation is written with an explicit
// round-to-nearest intrinsic and the library is built with -fmad=false, so no
// multiply-add is contracted behind our back):
//   FP16 row   : S^ = (float)h                         exact
//   INT8 row   : S^ = fl(code * scale)                 one rounding
//   requantize : FP16  h = RN16(x)  (cvt.rn, IEEE overflow to inf)
//                INT8  a = max|x| over the row; scale = fl(a/127);
//                      inv = fl(127/a); code = RNE(x*inv) taken from ONE fused
//                      multiply-add with 1.5*2^23 (exact RNE of the exact
//                      product, see quantize4); a == 0 or inv == inf -> 0.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "damp_internal.h"

namespace damp {

// ----------------------------------------------------------------------------
// PTX wrappers
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t tx) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar),
                 "r"(tx)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// try_wait with a suspend-time hint: a warp whose phase is not complete
// sleeps (up to the hint) instead of spinning and taking issue slots.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity), "r"(1000000u)
        : "memory");
    return ok != 0;
}
__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
// Every wait in the pipeline is bounded: after kWaitNs it gives up and the
// caller records DAMP_EFLAG_TIMEOUT instead of waiting forever.  The timer is
// read once every 64 tries.
constexpr uint64_t kWaitNs = 2000000000ull;  // 2 s
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  uint64_t limit_ns = kWaitNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_ns();
    for (uint32_t n = 1;; ++n) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((n & 63u) == 0 && global_ns() - t0 > limit_ns) return false;
    }
}

// global -> shared bulk copy completing on an mbarrier (no tensor map, no multicast)
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes,
                                         uint32_t bar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(dst),
        "l"(src), "r"(bytes), "r"(bar)
        : "memory");
}
// shared -> global bulk copy in a bulk async-group
__device__ __forceinline__ void bulk_s2g(void* dst, uint32_t src, uint32_t bytes) {
    asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(dst),
                 "r"(src), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() {
    asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
    asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
template <int N>
__device__ __forceinline__ void bulk_wait_all() {
    asm volatile("cp.async.bulk.wait_group %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void bar_sync(int id, int n) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}
// Barrier that also returns the OR of `pred` over the participating threads.
__device__ __forceinline__ int bar_red_or(int id, int n, int pred) {
    int r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.s32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.s32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(pred), "r"(id), "r"(n)
        : "memory");
    return r;
}

// ----------------------------------------------------------------------------
// Thread tile: a 256-thread group holds 128/d units; each unit's d x d state is
// spread over 2d threads as 8 row groups x (d/4) column groups.  A thread owns
// rows [r0, r0 + d/8) and columns [4*cg, 4*cg + 4).  The d/4 threads of a row
// group are consecutive lanes of one warp.
// ----------------------------------------------------------------------------
template <int D>
struct Geo {
    static constexpr int RPT = D / 8;     // rows per thread
    static constexpr int LPR = D / 4;     // lanes per row (column groups)
    static constexpr int UPI = 128 / D;   // units per 256-thread group
    static constexpr int TPU = 2 * D;     // threads per unit
    static_assert(D == 16 || D == 32 || D == 64 || D == 128, "d in {16,32,64,128}");
};

// FP16-row bits of rows [r0, r0 + RPT) and the rank of row r0 among FP16 rows.
// mask = the first 128 bits of the head's FP16-row mask (bit i = key row i is FP16).
template <int D>
__device__ __forceinline__ void row_formats(uint4 mask, int r0, uint32_t& bits, int& rank16) {
    constexpr int RPT = Geo<D>::RPT;
    const int w = r0 >> 5, sh = r0 & 31;
    const uint32_t word = (w == 0) ? mask.x : (w == 1) ? mask.y : (w == 2) ? mask.z : mask.w;
    rank16 = (w > 0 ? __popc(mask.x) : 0) + (w > 1 ? __popc(mask.y) : 0) +
             (w > 2 ? __popc(mask.z) : 0) + __popc(word & ((1u << sh) - 1u));
    bits = (word >> sh) & ((1u << RPT) - 1u);
}

__device__ __forceinline__ float2 f2(float a) { return make_float2(a, a); }

// Two FP32 products, each rounded to nearest even, as two scalar multiplies.
// (The d = 128 kernel forms the same products with the packed f32x2
// multiply, which rounds each half the same way; its states are checked
// bit for bit against these kernels and the oracle.)
__device__ __forceinline__ float2 mul2_rn(float2 a, float2 b) {
    return make_float2(__fmul_rn(a.x, b.x), __fmul_rn(a.y, b.y));
}

__device__ __forceinline__ void dequant_fp16x4(uint2 h, float2& lo, float2& hi) {
    lo = __half22float2(*reinterpret_cast<const __half2*>(&h.x));
    hi = __half22float2(*reinterpret_cast<const __half2*>(&h.y));
}

__device__ __forceinline__ uint2 quant_fp16x4(float2 lo, float2 hi) {
    __half2 a = __float22half2_rn(lo);
    __half2 b = __float22half2_rn(hi);
    uint2 r;
    r.x = *reinterpret_cast<uint32_t*>(&a);
    r.y = *reinterpret_cast<uint32_t*>(&b);
    return r;
}

// Codes of 4 values: RNE(x*inv).  fma(x, inv, 1.5*2^23) rounds the exact
// product plus 1.5*2^23 once; |x*inv| <= 127 + 2^-16 keeps the sum inside
// [2^23, 2^24) where the FP32 spacing is 1, so the rounding is to the nearest
// integer with ties to even, and the low byte of the result's bit pattern is
// the two's-complement code.  inv == 0 gives code 0.
__device__ __forceinline__ uint32_t quant_int8x4(float2 lo, float2 hi, float inv) {
    const float2 magic = f2(12582912.0f);
    const float2 a = __ffma2_rn(lo, f2(inv), magic);
    const float2 b = __ffma2_rn(hi, f2(inv), magic);
    const uint32_t p01 = __byte_perm(__float_as_uint(a.x), __float_as_uint(a.y), 0x0040);
    const uint32_t p23 = __byte_perm(__float_as_uint(b.x), __float_as_uint(b.y), 0x0040);
    return __byte_perm(p01, p23, 0x5410);
}

__device__ __forceinline__ float absmax4(float2 lo, float2 hi) {
    return fmaxf(fmaxf(fabsf(lo.x), fabsf(lo.y)), fmaxf(fabsf(hi.x), fabsf(hi.y)));
}

// Max over the d/4 lanes of a row group (all lanes get it).  d == 128 uses
// one warp-wide integer max (|x| >= 0 orders like its bit pattern).
template <int D>
__device__ __forceinline__ float rowgroup_max(float m) {
    if constexpr (D == 128) {
        return __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(m)));
    } else {
#pragma unroll
        for (int off = Geo<D>::LPR / 2; off >= 1; off >>= 1)
            m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, off));
        return m;
    }
}

// scale = fl(a/Q), inv = fl(Q/a) with Q = 127 (INT8 rows) or 448 (the largest
// finite FP8 E4M3 value); zero / overflowing rows -> 0, 0.
template <bool FP8 = false>
__device__ __forceinline__ void row_scale(float a, float& scale, float& inv) {
    constexpr float Q = FP8 ? 448.0f : 127.0f;
    inv = __fdiv_rn(Q, a);
    scale = __fdiv_rn(a, Q);
    if (a == 0.0f || isinf(inv)) {
        inv = 0.0f;
        scale = 0.0f;
    }
}

// fl(value(code) * s) for 4 FP8 E4M3 codes (byte j = element j).  Each pair
// of codes is widened exactly to two FP16 values (E4M3 is a subset of FP16),
// then to FP32, then scaled.
__device__ __forceinline__ void dequant_e4m3x4(uint32_t w, float s, float2& lo, float2& hi) {
    uint32_t h01, h23;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h01) : "h"((unsigned short)(w & 0xffffu)));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h23) : "h"((unsigned short)(w >> 16)));
    lo = mul2_rn(__half22float2(*reinterpret_cast<const __half2*>(&h01)), f2(s));
    hi = mul2_rn(__half22float2(*reinterpret_cast<const __half2*>(&h23)), f2(s));
}

// E4M3 codes of 4 values: the FP32 products x*inv converted to the nearest
// E4M3 value (ties to even), saturating at +-448.  The conversion puts its
// first source operand in the upper byte.
__device__ __forceinline__ uint32_t quant_e4m3x4(float2 lo, float2 hi, float inv) {
    const float2 a = mul2_rn(lo, f2(inv));
    const float2 b = mul2_rn(hi, f2(inv));
    unsigned short p01, p23;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(p01) : "f"(a.y), "f"(a.x));
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(p23) : "f"(b.y), "f"(b.x));
    // a row stored as zero (inv == 0) has code 0 everywhere: x * 0 is -0 for
    // negative x, whose E4M3 code would be 0x80
    return inv == 0.0f ? 0u : ((uint32_t)p01 | ((uint32_t)p23 << 16));
}

// Requantize rows [r0, r0+RPT) of x into a quantized block at `blk` (shared or
// global).  rowbuf: 2*RPT floats private to this row group (shared memory).
// Must be called by every lane of the warp (it synchronises the warp).
template <int D, bool FP8 = false>
__device__ __forceinline__ void store_quant_tile(uint8_t* blk, uint32_t f16_off, uint32_t i8_off,
                                                 uint32_t bits, int rank16, int r0, int cg,
                                                 const float2 (&x)[Geo<D>::RPT][2],
                                                 float* rowbuf) {
    constexpr int RPT = Geo<D>::RPT;
    float amax[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        amax[i] = 0.0f;
        if (D < 128 || !((bits >> i) & 1u)) amax[i] = rowgroup_max<D>(absmax4(x[i][0], x[i][1]));
    }
    // lane cg == 0 publishes the row maxima; lane cg < RPT takes row cg
    if (cg == 0) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) rowbuf[i] = amax[i];
    }
    __syncwarp();
    if (cg < RPT && !((bits >> cg) & 1u)) {
        float scale, inv;
        row_scale<FP8>(rowbuf[cg], scale, inv);
        rowbuf[RPT + cg] = inv;
        const int rank8 = r0 + cg - rank16 - __popc(bits & ((1u << cg) - 1u));
        *reinterpret_cast<float*>(blk + (size_t)rank8 * 4) = scale;
    }
    __syncwarp();
    int r16 = rank16, r8 = r0 - rank16;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        if ((bits >> i) & 1u) {
            const uint2 h = quant_fp16x4(x[i][0], x[i][1]);
            uint8_t* row = blk + f16_off + (size_t)r16 * (2 * D);
            *reinterpret_cast<uint32_t*>(row + cg * 4) = h.x;
            *reinterpret_cast<uint32_t*>(row + D + cg * 4) = h.y;
            ++r16;
        } else {
            *reinterpret_cast<uint32_t*>(blk + i8_off + (size_t)r8 * D + cg * 4) =
                FP8 ? quant_e4m3x4(x[i][0], x[i][1], rowbuf[RPT + i])
                    : quant_int8x4(x[i][0], x[i][1], rowbuf[RPT + i]);
            ++r8;
        }
    }
    __syncwarp();  // rowbuf may be reused by the caller's next tile
}

// ---------------------------------------------------------------------------
// Shared-memory variants for the decode step, addressed through the head's
// row directory (one word per key row: row offset, scale offset, FP16 flag).
// The block sits in a pipeline stage followed by at least 256 more bytes of
// the same allocation, so both candidate reads of a row (the FP16 row's two
// plane words, the byte row's word, which is the first of them, and the
// scale) are always in bounds and can be issued unconditionally: no load waits on a branch, and the rows' dependency chains
// overlap.  Stores are made per the row's format.
// ---------------------------------------------------------------------------

// fl(code * scale) for 4 INT8 codes.  Each code, biased to 1..255, is placed
// in the low mantissa bits of 2^23 by a byte permute; one exact packed
// subtraction of 2^23 + 128 recovers the code and one packed multiply
// applies the scale.  (Converting each byte with an integer-to-float
// instruction measured ~5 % slower: those run on the quarter-rate
// conversion pipe.)
__device__ __forceinline__ void dequant_int8x4_packed(uint32_t w, float s, float2& lo, float2& hi) {
    const uint32_t wb = w ^ 0x80808080u;
    const float2 bias = f2(-8388736.0f);  // -(2^23 + 128)
    float2 c01 = make_float2(__uint_as_float(__byte_perm(wb, 0x4B000000u, 0x7440)),
                             __uint_as_float(__byte_perm(wb, 0x4B000000u, 0x7441)));
    float2 c23 = make_float2(__uint_as_float(__byte_perm(wb, 0x4B000000u, 0x7442)),
                             __uint_as_float(__byte_perm(wb, 0x4B000000u, 0x7443)));
    c01 = __fadd2_rn(c01, bias);
    c23 = __fadd2_rn(c23, bias);
    lo = __fmul2_rn(c01, f2(s));
    hi = __fmul2_rn(c23, f2(s));
}

// Rows [r0, r0+RPT) x cols [4cg, 4cg+4) of a quantized block in global memory,
// located from the row-format bits of the thread's rows (bit i: row r0 + i is
// FP16) and rank16 (FP16 rows below r0), as store_quant_tile does: no load
// waits on another, so every row's reads are in flight together.
template <int D, bool FP8 = false>
__device__ __forceinline__ void load_tile_mask(const uint8_t* blk, uint32_t f16_off, uint32_t i8_off,
                                               uint32_t bits, int rank16, int r0, int cg,
                                               float2 (&x)[Geo<D>::RPT][2]) {
    constexpr int RPT = Geo<D>::RPT;
    uint2 raw[RPT];   // FP16 row: its two plane words; byte row: 4 codes in .x, the row's scale in .y
    int r16 = rank16, r8 = r0 - rank16;
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        if ((bits >> i) & 1u) {
            const uint8_t* row = blk + f16_off + (size_t)r16 * (2 * D);
            raw[i].x = __ldg(reinterpret_cast<const uint32_t*>(row + cg * 4));
            raw[i].y = __ldg(reinterpret_cast<const uint32_t*>(row + D + cg * 4));
            ++r16;
        } else {
            raw[i].x = __ldg(reinterpret_cast<const uint32_t*>(blk + i8_off + (size_t)r8 * D + cg * 4));
            raw[i].y = __ldg(reinterpret_cast<const uint32_t*>(blk + (size_t)r8 * 4));
            ++r8;
        }
    }
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        if ((bits >> i) & 1u) dequant_fp16x4(raw[i], x[i][0], x[i][1]);
        else if constexpr (FP8) dequant_e4m3x4(raw[i].x, __uint_as_float(raw[i].y), x[i][0], x[i][1]);
        else dequant_int8x4_packed(raw[i].x, __uint_as_float(raw[i].y), x[i][0], x[i][1]);
    }
}

// max(|a|, |b|, |c|, |d|) with a three-input maximum
__device__ __forceinline__ float absmax4_3(float2 lo, float2 hi) {
    float m;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(fabsf(lo.x)), "f"(fabsf(lo.y)), "f"(fabsf(hi.x)));
    return fmaxf(m, fabsf(hi.y));
}

template <int D, bool FP8 = false>
__device__ __forceinline__ void load_tile_dir(const uint8_t* blk, const uint32_t* dir, int r0,
                                              int cg, float2 (&x)[Geo<D>::RPT][2]) {
    constexpr int RPT = Geo<D>::RPT;
    constexpr int BATCH = RPT < 8 ? RPT : 8;
#pragma unroll
    for (int i0 = 0; i0 < RPT; i0 += BATCH) {
        uint32_t e[BATCH];
        uint2 w16[BATCH];
        uint32_t w8[BATCH];
        float sc[BATCH];
#pragma unroll
        for (int j = 0; j < BATCH; ++j) {
            e[j] = dir[r0 + i0 + j];
            const uint8_t* row = blk + dir_row(e[j]);
            w8[j] = *reinterpret_cast<const uint32_t*>(row + cg * 4);
            w16[j] = make_uint2(w8[j], *reinterpret_cast<const uint32_t*>(row + D + cg * 4));
            sc[j] = *reinterpret_cast<const float*>(blk + dir_scale(e[j]));
        }
#pragma unroll
        for (int j = 0; j < BATCH; ++j) {
            if (e[j] >> 31) dequant_fp16x4(w16[j], x[i0 + j][0], x[i0 + j][1]);
            else if constexpr (FP8) dequant_e4m3x4(w8[j], sc[j], x[i0 + j][0], x[i0 + j][1]);
            else dequant_int8x4_packed(w8[j], sc[j], x[i0 + j][0], x[i0 + j][1]);
        }
    }
}

template <int D, bool FP8 = false>
__device__ __forceinline__ void store_tile_dir(uint8_t* blk, const uint32_t* dir, int r0, int cg,
                                               const float2 (&x)[Geo<D>::RPT][2],
                                               float* rowbuf) {
    constexpr int RPT = Geo<D>::RPT;
    float amax[RPT];
#pragma unroll
    for (int i = 0; i < RPT; ++i) amax[i] = rowgroup_max<D>(absmax4_3(x[i][0], x[i][1]));
    if (cg == 0) {
#pragma unroll
        for (int i = 0; i < RPT; ++i) rowbuf[i] = amax[i];
    }
    __syncwarp();
    if (cg < RPT) {
        const uint32_t e = dir[r0 + cg];
        if (!(e >> 31)) {
            float scale, inv;
            row_scale<FP8>(rowbuf[cg], scale, inv);
            rowbuf[RPT + cg] = inv;
            *reinterpret_cast<float*>(blk + dir_scale(e)) = scale;
        }
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < RPT; ++i) {
        const uint32_t e = dir[r0 + i];
        uint8_t* row = blk + dir_row(e);
        if (e >> 31) {
            const uint2 h = quant_fp16x4(x[i][0], x[i][1]);
            *reinterpret_cast<uint32_t*>(row + cg * 4) = h.x;
            *reinterpret_cast<uint32_t*>(row + D + cg * 4) = h.y;
        } else {
            *reinterpret_cast<uint32_t*>(row + cg * 4) =
                FP8 ? quant_e4m3x4(x[i][0], x[i][1], rowbuf[RPT + i])
                    : quant_int8x4(x[i][0], x[i][1], rowbuf[RPT + i]);
        }
    }
    __syncwarp();
}

}  // namespace damp
