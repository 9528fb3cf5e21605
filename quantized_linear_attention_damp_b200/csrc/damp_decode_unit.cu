// damp_decode_unit.cu -- decode step for quantized d = 128 states, one unit
// (slot, head) per CTA iteration, two CTAs per SM.
//
// Same arithmetic, same order of operations and same results as the generic
// kernel in damp_decode.cu ("STEPQuant ...", Appendix Table C2 steps 1, 2,
// 3, 6 on the DAMP row format); only the work decomposition differs.
//
// CTA of 8 warps.  Warp w owns key rows [16w, 16w + 16) of the unit and lane
// l owns columns [4l, 4l + 4), so every instruction of a warp works on one key
// row (or one pair of rows): format branches are uniform over the warp, only
// the bytes a row's format stores are read, and a row maximum is one
// warp-wide reduction.  Rows 2p and 2p + 1 of the warp share one packed FP32
// register pair per column (.x = row 2p, .y = row 2p + 1), so the per-row
// operands of the packed operations (scale, decay, k, q, beta*k, 1/scale)
// are natural pairs, and the first level of the pairwise sum u = k^T S' is
// the horizontal add of one packed product.  Each thread keeps its 16 x 4
// tile in registers from dequantize to requantize.  u is summed in the
// recursive pairwise order: 16 rows per thread as a subtree (levels 1-4),
// then the top three levels over the 8 warps.
//
// Per-row operands are gathered once per unit into a small table per warp
// (k, q, beta*k, the row scale, the dequantization offset, the row's offset
// in the block, the KDA decay), by half of the warp's lanes, one row each.
// A row's words are loaded from wherever its format keeps them, outside any
// branch, so that the loads of later rows can be issued ahead; the decode,
// and later the store, are inline PTX with a branch on the row's format
// marked bra.uni: the format is the same in every lane, so the branch needs
// no reconvergence.  A pair of byte rows is stored behind one test.  Pools
// of INT8 rows only or E4M3 rows only have their own instantiation, with no
// format test at all.
//
// Two CTAs share an SM whenever three stages fit in half of its shared
// memory (4 stages at 27 FP16 rows): their barriers are independent, so one
// CTA's arithmetic fills the other's barrier waits.  An item needs one CTA
// barrier: after it, every warp combines the 8 warps' partial sums for its
// own lanes' columns (the same values in every warp, so no second barrier;
// the partials are double-buffered by item parity, so a warp that starts
// the next item cannot overwrite them while another still reads them).
// Meanwhile warp 6 writes back the previous unit's block (one bulk store,
// once the barrier has ordered every writer's fenced rows before it) and the
// two warps refill the pipeline: cp.async.bulk copies into a shared-memory
// ring of stages completing on mbarriers (no tensor map, no multicast), two
// arrivals per stage: warp 7 copies the block and the head's row directory,
// warp 6 the unit's q, k, v and KDA decays.  Warp 6 waits for the stage's old
// store to have read it before it arrives at the item's barrier, so after
// the barrier both may reuse it.  The refill sits on every item's critical
// path (the next barrier waits for these warps), so it is kept short and
// split between them: each lane of warp 7 holds the metadata of every 32nd
// unit, loaded 32 units ahead with a division-free cursor, and the lane that
// holds an item issues its copies itself; warp 6 needs only the unit index.

#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <mutex>

#include "damp.h"
#include "damp_device.cuh"

namespace damp {
namespace {

constexpr int kPT = 256;       // threads (8 warps)
constexpr int kPD = 128;       // d_k = d_v
constexpr int kRW = 16;        // key rows per warp
constexpr int kPP = kRW / 2;   // row pairs per warp
constexpr int kNW = kPT / 32;  // warps
constexpr uint32_t kDirBytes = kPD * 4;   // the head's row directory
// Row formats of a pool: FP16 and INT8 rows (per the directory), INT8 rows
// only, or E4M3 rows only (no format test per row in the last two).
constexpr int kRowsMixed = 0, kRowsInt8 = 1, kRowsFp8 = 2;

// Per-unit metadata written by the refill warp into the stage (32 bytes).
struct PMeta {
    int active;        // 1: block loaded, to be updated and stored
    uint32_t bytes;    // block size of the unit's head
    float alpha;       // GDN scalar decay
    float beta;
    long long unit;    // b*H + h: row of q/k/v/alpha/beta/out; -1: no such entry
    long long boff;    // byte offset of the block in the pool; -1 if none
};
static_assert(sizeof(PMeta) == 32, "PMeta layout");

// Per-warp table of the warp's 16 rows, as pairs (rows 2p, 2p + 1).
// The entries read only before the item's barrier (the decays and the
// dequantization offsets) share their space with those written only after it
// (the row maxima and inverse scales): a warp fills its table for the next
// item only after its last read of this item's.
struct RowTab {
    float4 kq[kPP];      // {k_2p, k_2p+1, q_2p, q_2p+1}
    float4 bs[kPP];      // {b_2p, b_2p+1, s_2p, s_2p+1}: b = beta*k; s = row scale (1 for FP16 rows)
    uint2 off[kPP];      // byte offsets of rows 2p, 2p+1 in the block
    union {
        float2 al[kPP];  // KDA decays of rows 2p, 2p+1 (phase A)
        float inv[kRW];  // Q / amax (byte rows; 0 for zero rows) (requantization)
    };
    union {
        float2 bz[kPP];  // dequantization offsets of rows 2p, 2p+1: -(2^23+128) byte rows, -0 FP16 rows (phase A)
        float amax[kRW]; // row maxima of |X| (byte rows) (requantization)
    };
    uint32_t soff[kRW];  // byte offset of each byte row's scale in the block
};
static_assert(sizeof(RowTab) % 16 == 0, "RowTab layout");

template <bool BF16>
__device__ __forceinline__ float in_at(const uint8_t* base, int idx) {
    if constexpr (BF16) {
        return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(base)[idx])
                               << 16);
    } else {
        return reinterpret_cast<const float*>(base)[idx];
    }
}

// The four E4M3 codes of w widened exactly to FP32 (E4M3 is a subset of FP16).
__device__ __forceinline__ void e4m3x4_to_f32(uint32_t w, float (&f)[4]) {
    uint32_t h01, h23;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h01) : "h"((unsigned short)(w & 0xffffu)));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h23) : "h"((unsigned short)(w >> 16)));
    const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&h01));
    const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&h23));
    f[0] = a.x; f[1] = a.y; f[2] = b.x; f[3] = b.y;
}

// A float2 held in one 64-bit register (the operand type of the packed FP32
// instructions) and back.
__device__ __forceinline__ float2 as_f2(unsigned long long v) {
    float2 r;
    asm("mov.b64 {%0, %1}, %2;" : "=f"(r.x), "=f"(r.y) : "l"(v));
    return r;
}
__device__ __forceinline__ unsigned long long as_u64(float2 v) {
    unsigned long long r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(v.x), "f"(v.y));
    return r;
}

// Both rows of a pair decoded and dequantized from their words, which the
// caller has loaded (rows 2p, 2p + 1 as .x, .y; FP16 flags = bits 2p and
// 2p + 1 of m): x[c] = fl((raw_c + bz) * s), raw = the exact binary16 value
// (FP16 row: both words) or 2^23 + 128 + code (byte row: the codes in the
// first word).  Each row's format is a uniform branch (bra.uni: the same in
// every lane); the offset and the scale are packed operations on the pair.
__device__ __forceinline__ void pair_decode(int P, uint32_t m, uint32_t we0, uint32_t we1,
                                            uint32_t wo0, uint32_t wo1, float2 bz, float2 sp,
                                            float2 (&x)[4]) {
    unsigned long long r0, r1, r2, r3;
    asm("{\n\t"
        ".reg .pred p, pe, po;\n\t"
        ".reg .b32 t, wb, e0, e1, e2, e3, d0, d1, d2, d3;\n\t"
        ".reg .b16 h0, h1, h2, h3;\n\t"
        "and.b32 t, %4, %10;\n\t"
        "setp.ne.u32 pe, t, 0;\n\t"
        "@pe bra.uni EF16;\n\t"
        "xor.b32 wb, %5, 0x80808080;\n\t"
        "prmt.b32 e0, wb, %9, 0x7440;\n\t"
        "prmt.b32 e1, wb, %9, 0x7441;\n\t"
        "prmt.b32 e2, wb, %9, 0x7442;\n\t"
        "prmt.b32 e3, wb, %9, 0x7443;\n\t"
        "bra.uni EEND;\n\t"
        "EF16:\n\t"
        "mov.b32 {h0, h1}, %5;\n\t"
        "mov.b32 {h2, h3}, %6;\n\t"
        "cvt.f32.f16 e0, h0;\n\t"
        "cvt.f32.f16 e1, h1;\n\t"
        "cvt.f32.f16 e2, h2;\n\t"
        "cvt.f32.f16 e3, h3;\n\t"
        "EEND:\n\t"
        "and.b32 t, %4, %11;\n\t"
        "setp.ne.u32 po, t, 0;\n\t"
        "@po bra.uni OF16;\n\t"
        "xor.b32 wb, %7, 0x80808080;\n\t"
        "prmt.b32 d0, wb, %9, 0x7440;\n\t"
        "prmt.b32 d1, wb, %9, 0x7441;\n\t"
        "prmt.b32 d2, wb, %9, 0x7442;\n\t"
        "prmt.b32 d3, wb, %9, 0x7443;\n\t"
        "bra.uni PEND;\n\t"
        "OF16:\n\t"
        "mov.b32 {h0, h1}, %7;\n\t"
        "mov.b32 {h2, h3}, %8;\n\t"
        "cvt.f32.f16 d0, h0;\n\t"
        "cvt.f32.f16 d1, h1;\n\t"
        "cvt.f32.f16 d2, h2;\n\t"
        "cvt.f32.f16 d3, h3;\n\t"
        "PEND:\n\t"
        "mov.b64 %0, {e0, d0};\n\t"
        "mov.b64 %1, {e1, d1};\n\t"
        "mov.b64 %2, {e2, d2};\n\t"
        "mov.b64 %3, {e3, d3};\n\t"
        "add.rn.f32x2 %0, %0, %12;\n\t"
        "add.rn.f32x2 %1, %1, %12;\n\t"
        "add.rn.f32x2 %2, %2, %12;\n\t"
        "add.rn.f32x2 %3, %3, %12;\n\t"
        "mul.rn.f32x2 %0, %0, %13;\n\t"
        "mul.rn.f32x2 %1, %1, %13;\n\t"
        "mul.rn.f32x2 %2, %2, %13;\n\t"
        "mul.rn.f32x2 %3, %3, %13;\n\t"
        "}"
        : "=l"(r0), "=l"(r1), "=l"(r2), "=l"(r3)
        : "r"(m), "r"(we0), "r"(we1), "r"(wo0), "r"(wo1), "r"(0x4B000000u),
          "r"(1u << (2 * P)), "r"(2u << (2 * P)), "l"(as_u64(bz)), "l"(as_u64(sp)));
    x[0] = as_f2(r0); x[1] = as_f2(r1); x[2] = as_f2(r2); x[3] = as_f2(r3);
}

// Two byte rows of a pair decoded and dequantized (pools with no FP16 rows):
// x[c] = fl((2^23 + 128 + code_c - (2^23 + 128)) * s) for row 2p (.x, codes
// in we) and row 2p + 1 (.y, codes in wo).
__device__ __forceinline__ void pair_decode_i8(uint32_t we, uint32_t wo, float2 sp, float2 (&x)[4]) {
    unsigned long long r0, r1, r2, r3;
    asm("{\n\t"
        ".reg .b32 wb, vb, e0, e1, e2, e3, d0, d1, d2, d3;\n\t"
        ".reg .b64 bz;\n\t"
        "xor.b32 wb, %4, 0x80808080;\n\t"
        "xor.b32 vb, %5, 0x80808080;\n\t"
        "prmt.b32 e0, wb, %6, 0x7440;\n\t"
        "prmt.b32 e1, wb, %6, 0x7441;\n\t"
        "prmt.b32 e2, wb, %6, 0x7442;\n\t"
        "prmt.b32 e3, wb, %6, 0x7443;\n\t"
        "prmt.b32 d0, vb, %6, 0x7440;\n\t"
        "prmt.b32 d1, vb, %6, 0x7441;\n\t"
        "prmt.b32 d2, vb, %6, 0x7442;\n\t"
        "prmt.b32 d3, vb, %6, 0x7443;\n\t"
        "mov.b64 %0, {e0, d0};\n\t"
        "mov.b64 %1, {e1, d1};\n\t"
        "mov.b64 %2, {e2, d2};\n\t"
        "mov.b64 %3, {e3, d3};\n\t"
        "mov.b64 bz, {%7, %7};\n\t"
        "add.rn.f32x2 %0, %0, bz;\n\t"
        "add.rn.f32x2 %1, %1, bz;\n\t"
        "add.rn.f32x2 %2, %2, bz;\n\t"
        "add.rn.f32x2 %3, %3, bz;\n\t"
        "mul.rn.f32x2 %0, %0, %8;\n\t"
        "mul.rn.f32x2 %1, %1, %8;\n\t"
        "mul.rn.f32x2 %2, %2, %8;\n\t"
        "mul.rn.f32x2 %3, %3, %8;\n\t"
        "}"
        : "=l"(r0), "=l"(r1), "=l"(r2), "=l"(r3)
        : "r"(we), "r"(wo), "r"(0x4B000000u), "r"(0xCB000080u), "l"(as_u64(sp)));
    x[0] = as_f2(r0); x[1] = as_f2(r1); x[2] = as_f2(r2); x[3] = as_f2(r3);
}

// Store both rows of a pair at their words a_e, a_o: the two code words when
// both are byte rows (one uniform test), else row by row (byte row -> its
// code word; FP16 row -> its four values rounded to binary16, one word in
// each plane).
__device__ __forceinline__ void pair_store(int P, uint32_t m, uint32_t ae, uint32_t ao, uint2 cw,
                                           const float2 (&x)[4]) {
    asm volatile("{\n\t"
        ".reg .pred p, pe, po;\n\t"
        ".reg .b32 t, h01, h23;\n\t"
        "and.b32 t, %0, %13;\n\t"
        "setp.ne.u32 p, t, 0;\n\t"
        "@p bra.uni QMIX;\n\t"
        "st.shared.u32 [%1], %3;\n\t"
        "st.shared.u32 [%2], %4;\n\t"
        "bra.uni QEND;\n\t"
        "QMIX:\n\t"
        "and.b32 t, %0, %14;\n\t"
        "setp.ne.u32 pe, t, 0;\n\t"
        "@pe bra.uni QEF;\n\t"
        "st.shared.u32 [%1], %3;\n\t"
        "bra.uni QEE;\n\t"
        "QEF:\n\t"
        "cvt.rn.f16x2.f32 h01, %6, %5;\n\t"
        "cvt.rn.f16x2.f32 h23, %8, %7;\n\t"
        "st.shared.u32 [%1], h01;\n\t"
        "st.shared.u32 [%1+128], h23;\n\t"
        "QEE:\n\t"
        "and.b32 t, %0, %15;\n\t"
        "setp.ne.u32 po, t, 0;\n\t"
        "@po bra.uni QOF;\n\t"
        "st.shared.u32 [%2], %4;\n\t"
        "bra.uni QEND;\n\t"
        "QOF:\n\t"
        "cvt.rn.f16x2.f32 h01, %10, %9;\n\t"
        "cvt.rn.f16x2.f32 h23, %12, %11;\n\t"
        "st.shared.u32 [%2], h01;\n\t"
        "st.shared.u32 [%2+128], h23;\n\t"
        "QEND:\n\t"
        "}"
        :: "r"(m), "r"(ae), "r"(ao), "r"(cw.x), "r"(cw.y),
           "f"(x[0].x), "f"(x[1].x), "f"(x[2].x), "f"(x[3].x),
           "f"(x[0].y), "f"(x[1].y), "f"(x[2].y), "f"(x[3].y),
           "r"(3u << (2 * P)), "r"(1u << (2 * P)), "r"(2u << (2 * P))
        : "memory");
}

// max |v| over 4 values
__device__ __forceinline__ float absmax4v(float a, float b, float c, float d) {
    return fmaxf(fmaxf(fabsf(a), fabsf(b)), fmaxf(fabsf(c), fabsf(d)));
}

// Two byte rows at once (inverse scales as a pair).
template <bool FP8>
__device__ __forceinline__ uint2 quant_pair4(const float2 (&x)[4], float2 inv) {
    if constexpr (FP8) {
        float2 y[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) y[c] = __fmul2_rn(x[c], inv);
        unsigned short e01, e23, o01, o23;
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(e01) : "f"(y[1].x), "f"(y[0].x));
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(e23) : "f"(y[3].x), "f"(y[2].x));
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(o01) : "f"(y[1].y), "f"(y[0].y));
        asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(o23) : "f"(y[3].y), "f"(y[2].y));
        // rows stored as zero (inv == 0) have code 0 (not the -0 code 0x80)
        return make_uint2(inv.x == 0.0f ? 0u : ((uint32_t)e01 | ((uint32_t)e23 << 16)),
                          inv.y == 0.0f ? 0u : ((uint32_t)o01 | ((uint32_t)o23 << 16)));
    } else {
        // RNE of the exact x*inv by one fused multiply-add with 1.5*2^23 (the
        // low byte of the sum is the two's-complement code; see quant_int8x4)
        const float2 magic = f2(12582912.0f);
        float2 y[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) y[c] = __ffma2_rn(x[c], inv, magic);
        const uint32_t e01 = __byte_perm(__float_as_uint(y[0].x), __float_as_uint(y[1].x), 0x0040);
        const uint32_t e23 = __byte_perm(__float_as_uint(y[2].x), __float_as_uint(y[3].x), 0x0040);
        const uint32_t o01 = __byte_perm(__float_as_uint(y[0].y), __float_as_uint(y[1].y), 0x0040);
        const uint32_t o23 = __byte_perm(__float_as_uint(y[2].y), __float_as_uint(y[3].y), 0x0040);
        return make_uint2(__byte_perm(e01, e23, 0x5410), __byte_perm(o01, o23, 0x5410));
    }
}

template <bool KDA, bool BF16, int ROWS>
__global__ void __launch_bounds__(kPT, 2) decode_unit_kernel(const StepArgs a) {
    constexpr bool FP8 = ROWS == kRowsFp8, I8 = ROWS == kRowsInt8;
    constexpr uint32_t ELT = BF16 ? 2 : 4;
    constexpr float kQ = FP8 ? 448.0f : 127.0f;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int NS = a.n_stages;
    const uint32_t bar0 = smem_u32(smem + a.bar_off);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(full_bar(s), 2);
        fence_mbar_init();
    }
    __syncthreads();

    const int H = a.H;
    const int my_items = (a.n_items - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;

    // ---- refill side (warp 7): lane L holds the metadata of CTA-local unit
    // U == L (mod 32), loaded 32 units ahead of use.  The ring holds raw
    // values: nothing waits for the loads until the unit is issued, and no
    // branch depends on a freshly loaded slot index.
    constexpr int kIssueWarp = kNW - 1;         // refill: metadata, block, directory
    constexpr int kStoreWarp = kIssueWarp - 1;  // write-back; refill: q, k, v, KDA decays
    struct RMeta {
        int slot;          // slot index; INT_MIN: no such unit
        float alpha, beta;
        int unit;
        int head;
        uint2 hb;          // the head's {block offset in the slot, block size}
    };
    // Lane L of the refill warp loads the units U = L, L + 32, L + 64, ... of
    // this CTA (unit u = blockIdx + U * gridDim = b * H + h): it keeps (u, b, h)
    // of its next unit and advances them by 32 * gridDim units each time, so
    // no load needs a division.
    const int du = 32 * (int)gridDim.x, db = du / H, dh = du - db * H;
    int nu = (int)blockIdx.x + lane * (int)gridDim.x;
    int nb = nu / H, nh = nu - nb * H;
    auto load_meta = [&](int U) {
        RMeta r{INT_MIN, 0.f, 0.f, -1, 0, make_uint2(0u, 0u)};
        if (U < my_items) {
            r.head = nh;
            r.slot = __ldg(a.slot_idx + nb);
            r.unit = nu;
            if constexpr (!KDA) r.alpha = __ldg(a.alpha + nu);
            r.beta = __ldg(a.beta + nu);
            r.hb = __ldg(reinterpret_cast<const uint2*>(a.heads + nh));
        }
        nu += du;
        nb += db;
        nh += dh;
        if (nh >= H) {
            nh -= H;
            ++nb;
        }
        return r;
    };
    // Stage metadata of a unit from its raw ring values.
    auto finish_meta = [&](const RMeta& r) {
        PMeta m{0, 0u, r.alpha, r.beta, -1, -1};
        if (r.slot != INT_MIN) {
            m.unit = r.unit;
            if (r.slot >= 0 && r.slot < a.n_slots) {
                m.active = 1;
                m.bytes = r.hb.y;
                m.boff = (long long)r.slot * (long long)a.slot_stride + r.hb.x;
            } else if (r.slot >= a.n_slots) {
                m.active = -1;   // out of range: flagged by the consumer
            }
        }
        return m;
    };
    RMeta ring{INT_MIN, 0.f, 0.f, -1, 0, make_uint2(0u, 0u)};
    if (warp == kIssueWarp) ring = load_meta(lane);

    // Programmatic dependent launch: everything above touches only this
    // call's inputs (slot indices, gates, the pool's block table), which no
    // earlier decode step writes, so it overlaps the previous kernel's tail.
    // From here on the pool, q/k/v and out are read or written: wait until the
    // grids this launch depends on have completed and their writes are
    // visible.  The next launch on the stream may start its own prologue now.
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;");

    // The refill warp's part of item il: the stage's metadata, the block and
    // the head's row directory (bulk copies completing on the stage's
    // mbarrier, issued by the lane that holds the item's metadata); q, k, v
    // and the KDA decays come from the store warp (issue_inputs).
    auto issue = [&](int il) {
        const int stage = il % NS;
        uint8_t* st = smem + (size_t)stage * a.stage_bytes;
        // the lane that holds the item's metadata issues it (no shuffles)
        if (lane == (il & 31)) {
            const PMeta m = finish_meta(ring);
            const int head = ring.head;
            if (!(il == 0 && (a.hooks & kHookHoldFirstItem))) {
                *reinterpret_cast<PMeta*>(st + a.st_meta) = m;
                const uint32_t fb = full_bar(stage);
                if (m.active == 1) {
                    mbar_arrive_expect_tx(fb, m.bytes + kDirBytes);
                    bulk_g2s(smem_u32(st), a.blocks + m.boff, m.bytes, fb);
                    bulk_g2s(smem_u32(st + a.st_dir), a.dir + (size_t)head * kPD, kDirBytes, fb);
                } else {
                    mbar_arrive(fb);
                }
            }
            ring = load_meta(il + 32);
        }
        __syncwarp();
    };

    // The inputs of item il (store warp, lane 0): q, k, v and the KDA decays
    // of unit blockIdx + il * gridDim, the stage's second arrival.
    auto issue_inputs = [&](int il) {
        const int stage = il % NS;
        uint8_t* st = smem + (size_t)stage * a.stage_bytes;
        const uint32_t fb = full_bar(stage);
        const size_t u = (size_t)blockIdx.x + (size_t)il * gridDim.x;
        const size_t io = u * kPD * ELT;
        mbar_arrive_expect_tx(fb, 3u * kPD * ELT + (KDA ? 4u * kPD : 0u));
        bulk_g2s(smem_u32(st + a.st_q), static_cast<const uint8_t*>(a.q) + io, kPD * ELT, fb);
        bulk_g2s(smem_u32(st + a.st_k), static_cast<const uint8_t*>(a.k) + io, kPD * ELT, fb);
        bulk_g2s(smem_u32(st + a.st_v), static_cast<const uint8_t*>(a.v) + io, kPD * ELT, fb);
        if constexpr (KDA) bulk_g2s(smem_u32(st + a.st_alpha), a.alpha + u * kPD, kPD * 4, fb);
    };

    // One bulk store of item j's block (store warp, lane 0).
    auto store_item = [&](int j) {
        const uint8_t* sj = smem + (size_t)(j % NS) * a.stage_bytes;
        const PMeta m = *reinterpret_cast<const PMeta*>(sj + a.st_meta);
        if (m.active == 1) bulk_s2g(a.blocks + m.boff, smem_u32(sj), m.bytes);
        bulk_commit();
    };

    const int ahead = NS - 2;
    int issued = 0;   // items issued so far (meaningful in the refill warp)
    if (warp == kIssueWarp)
        for (; issued < ahead && issued < my_items; ++issued) issue(issued);
    if (warp == kStoreWarp && lane == 0)
        for (int il = 0; il < ahead && il < my_items; ++il) issue_inputs(il);

    // ---- consumers: warp w owns rows [16w, 16w + 16), lane l columns [4l, 4l + 4)
    uint8_t* scratch = smem + a.scratch_off;
    float* red_u = reinterpret_cast<float*>(scratch);   // [2][8][128], by warp
    // per-warp partial sums, double-buffered by item parity: a warp may start
    // the next item while others still read this item's partials
    float* red_w = red_u + 2 * kNW * kPD;               // [2][8][128], by warp
    float* cprod = red_w + 2 * kNW * kPD;               // [2][128]: fl(q_i beta k_i) by row
    RowTab* tab = reinterpret_cast<RowTab*>(cprod + 2 * kPD) + warp;
    const int row0 = warp * kRW;

    int it = 0, stage = 0;
    uint32_t parity = 0;
    bool aborted = false;
    for (; it < my_items; ++it) {
        // A warp whose wait gave up in any lane skips the unit; the CTA leaves
        // the loop together at the first barrier below.
        const bool ok =
            __all_sync(0xffffffffu, mbar_wait_bounded(full_bar(stage), parity, a.wait_ns));
        uint8_t* st = smem + (size_t)stage * a.stage_bytes;
        const PMeta meta = *reinterpret_cast<const PMeta*>(st + a.st_meta);
        const bool any = ok && meta.active == 1;   // uniform over the warp
        uint8_t* blk = st;
        const uint8_t* sq = st + a.st_q;
        const uint8_t* sk = st + a.st_k;
        const uint32_t* sdir = reinterpret_cast<const uint32_t*>(st + a.st_dir);
        const uint8_t* b4 = blk + 4 * lane;   // this lane's 4 codes of a byte row
        // an FP16 row keeps this lane's 4 values as two words, at b4 and at
        // b4 + 128 (its two planes)

        float2 x[kPP][4];
        uint32_t m16 = 0;   // bit i: row row0 + i is an FP16 row
        if (any) {
            // ---- per-row operands of this warp's 16 rows (lanes 0-15, one row each)
            {
                bool f16 = false;
                if (lane < kRW) {
                    const int r = row0 + lane;
                    const uint32_t e = sdir[r];
                    f16 = (e >> 31) != 0;
                    const float kr = in_at<BF16>(sk, r), qr = in_at<BF16>(sq, r);
                    const float br = __fmul_rn(meta.beta, kr);
                    const uint32_t so = dir_scale(e);
                    const float sr = f16 ? 1.0f : *reinterpret_cast<const float*>(blk + so);
                    const int p = lane >> 1, j = lane & 1;
                    float* kq = reinterpret_cast<float*>(&tab->kq[p]);
                    float* bs = reinterpret_cast<float*>(&tab->bs[p]);
                    kq[j] = kr;
                    kq[2 + j] = qr;
                    bs[j] = br;
                    bs[2 + j] = sr;
                    reinterpret_cast<uint32_t*>(&tab->off[p])[j] = dir_row(e);
                    reinterpret_cast<float*>(&tab->bz[p])[j] = f16 ? -0.0f : -8388736.0f;
                    if constexpr (KDA)
                        reinterpret_cast<float*>(&tab->al[p])[j] =
                            reinterpret_cast<const float*>(st + a.st_alpha)[r];
                    tab->soff[lane] = so;
                    // this row's term of c = q^T (beta k), summed by the warp that writes out
                    cprod[(it & 1) * kPD + r] = __fmul_rn(qr, br);
                }
                m16 = __ballot_sync(0xffffffffu, f16);
                __syncwarp();
            }
            // ---- step 1 (reconstruct) and step 2 (first half), pair by pair:
            // S' = D S^; u = k^T S' (pairwise); w = q^T S'
            const float2 al_g = f2(meta.alpha);
            float2 wacc[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) wacc[c] = f2(0.f);
            float2 stk[3][2];
            float2 usum[2];
#pragma unroll
            for (int p = 0; p < kPP; ++p) {
                const uint2 o = tab->off[p];
                const float4 bs = tab->bs[p];
                const float2 sp = make_float2(bs.z, bs.w);
                if constexpr (I8) {
                    // INT8 pools hold no FP16 rows: both rows are INT8 rows
                    pair_decode_i8(*reinterpret_cast<const uint32_t*>(b4 + o.x),
                                   *reinterpret_cast<const uint32_t*>(b4 + o.y), sp, x[p]);
                } else if constexpr (!FP8) {
                    // each row's words (a byte row's word, or an FP16 row's
                    // two plane words; a byte row also reads the word 128
                    // bytes on, inside the stage, and does not use it),
                    // loaded outside the format branches so that they can be
                    // issued ahead; then the decode
                    const uint32_t* pe = reinterpret_cast<const uint32_t*>(b4 + o.x);
                    const uint32_t* po = reinterpret_cast<const uint32_t*>(b4 + o.y);
                    pair_decode(p, m16, pe[0], pe[kPD / 4], po[0], po[kPD / 4], tab->bz[p], sp, x[p]);
                } else {
                    // FP8 pools hold no FP16 rows: both rows are E4M3 rows
                    float e[4], d[4];
                    e4m3x4_to_f32(*reinterpret_cast<const uint32_t*>(b4 + o.x), e);
                    e4m3x4_to_f32(*reinterpret_cast<const uint32_t*>(b4 + o.y), d);
#pragma unroll
                    for (int c = 0; c < 4; ++c) x[p][c] = __fmul2_rn(make_float2(e[c], d[c]), sp);
                }
                const float2 alp = KDA ? tab->al[p] : al_g;
                const float4 kq = tab->kq[p];
                const float2 kp = make_float2(kq.x, kq.y), qp = make_float2(kq.z, kq.w);
                float L[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    x[p][c] = __fmul2_rn(x[p][c], alp);
                    const float2 pr = __fmul2_rn(kp, x[p][c]);   // fl(k_i S'_ij), two rows
                    L[c] = __fadd_rn(pr.x, pr.y);                  // level 1 of the pairwise sum
                    wacc[c] = __ffma2_rn(qp, x[p][c], wacc[c]);
                }
                float2 v[2] = {make_float2(L[0], L[1]), make_float2(L[2], L[3])};
#pragma unroll
                for (int lv = 0; lv < 3; ++lv) {   // levels 2-4 over this warp's pairs
                    if ((p >> lv) & 1) {
                        v[0] = __fadd2_rn(stk[lv][0], v[0]);
                        v[1] = __fadd2_rn(stk[lv][1], v[1]);
                    } else {
                        stk[lv][0] = v[0];
                        stk[lv][1] = v[1];
                        break;
                    }
                }
                if (p == kPP - 1) {
                    usum[0] = v[0];
                    usum[1] = v[1];
                }
            }
            reinterpret_cast<float4*>(red_u + ((it & 1) * kNW + warp) * kPD)[lane] =
                make_float4(usum[0].x, usum[0].y, usum[1].x, usum[1].y);
            reinterpret_cast<float4*>(red_w + ((it & 1) * kNW + warp) * kPD)[lane] =
                make_float4(__fadd_rn(wacc[0].x, wacc[0].y), __fadd_rn(wacc[1].x, wacc[1].y),
                            __fadd_rn(wacc[2].x, wacc[2].y), __fadd_rn(wacc[3].x, wacc[3].y));
        }
        // the store of item it-2 (issued a whole item ago) has read its stage
        // before the store warp arrives at the barrier, so after it the refill
        // warp may reuse that stage
        if (warp == kStoreWarp && lane == 0) bulk_wait_read<0>();
        if (bar_red_or(0, kPT, ok ? 0 : 1)) {
            aborted = true;
            break;
        }

        // ---- write back item it-1 (its requantized rows were fenced by their
        // writers before this barrier) and refill the stage of item it-2.
        if (warp == kStoreWarp) {
            if (lane == 0) {
                if (it + ahead < my_items) issue_inputs(it + ahead);
                if (it >= 1) store_item(it - 1);
            }
        } else if (warp == kIssueWarp) {
            if (it + ahead < my_items) {
                issue(it + ahead);
                issued = it + ahead + 1;
            }
        }
        // ---- step 2 (second half) + step 3, in every warp for its lanes'
        // columns 4l .. 4l+3: u by the top three pairwise levels over the 8
        // warps' partials, delta = v - u; w, c; warp 0 writes out.  Every warp
        // reads the same partials, so no second CTA barrier is needed.
        bool bad = false;   // a non-finite input (checked when a.validate)
        float2 dl[4];
        if (meta.active == 1) {
            const float* ru = red_u + (it & 1) * kNW * kPD;
            const float* rw = red_w + (it & 1) * kNW * kPD;
            float2 u01[2][4];   // [column pair][tree node]
#pragma unroll
            for (int q2 = 0; q2 < 4; ++q2) {
                const float4 a0 = reinterpret_cast<const float4*>(ru + (2 * q2) * kPD)[lane];
                const float4 a1 = reinterpret_cast<const float4*>(ru + (2 * q2 + 1) * kPD)[lane];
                u01[0][q2] = __fadd2_rn(make_float2(a0.x, a0.y), make_float2(a1.x, a1.y));
                u01[1][q2] = __fadd2_rn(make_float2(a0.z, a0.w), make_float2(a1.z, a1.w));
            }
            float2 uu[2];
#pragma unroll
            for (int h = 0; h < 2; ++h)
                uu[h] = __fadd2_rn(__fadd2_rn(u01[h][0], u01[h][1]), __fadd2_rn(u01[h][2], u01[h][3]));
            float vv[4];
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) vv[cc] = in_at<BF16>(st + a.st_v, 4 * lane + cc);
            // delta = fl(v - u) (the negation is exact)
            const float2 d01 = __fadd2_rn(make_float2(vv[0], vv[1]), make_float2(-uu[0].x, -uu[0].y));
            const float2 d23 = __fadd2_rn(make_float2(vv[2], vv[3]), make_float2(-uu[1].x, -uu[1].y));
            dl[0] = f2(d01.x);
            dl[1] = f2(d01.y);
            dl[2] = f2(d23.x);
            dl[3] = f2(d23.y);
            if (warp == 0) {
                // out = w + c delta (only this warp needs w and c)
                float2 ww[2] = {f2(0.f), f2(0.f)};
#pragma unroll
                for (int q2 = 0; q2 < kNW; ++q2) {
                    const float4 b0 = reinterpret_cast<const float4*>(rw + q2 * kPD)[lane];
                    ww[0] = __fadd2_rn(ww[0], make_float2(b0.x, b0.y));
                    ww[1] = __fadd2_rn(ww[1], make_float2(b0.z, b0.w));
                }
                const float4 c4 = reinterpret_cast<const float4*>(cprod + (it & 1) * kPD)[lane];
                float c = (c4.x + c4.y) + (c4.z + c4.w);   // c = q^T (beta k), any order
#pragma unroll
                for (int off = 16; off >= 1; off >>= 1) c += __shfl_xor_sync(0xffffffffu, c, off);
                const float2 o01 = __ffma2_rn(f2(c), d01, ww[0]);
                const float2 o23 = __ffma2_rn(f2(c), d23, ww[1]);
                reinterpret_cast<float4*>(a.out + (size_t)meta.unit * kPD)[lane] =
                    make_float4(o01.x, o01.y, o23.x, o23.y);
            }
            if (a.validate) {
                // every warp checks the same inputs: the vote is uniform over the CTA
                bool f = isfinite(meta.beta) && isfinite(meta.alpha);
#pragma unroll
                for (int cc = 0; cc < 4; ++cc) {
                    const int j = 4 * lane + cc;
                    f = f && isfinite(vv[cc]) && isfinite(in_at<BF16>(sq, j)) && isfinite(in_at<BF16>(sk, j));
                    if constexpr (KDA) f = f && isfinite(reinterpret_cast<const float*>(st + a.st_alpha)[j]);
                }
                bad = __any_sync(0xffffffffu, !f);
                if (bad) {
                    // the unit is skipped: out row zeroed, block neither updated nor stored
                    if (warp == 0) reinterpret_cast<float4*>(a.out + (size_t)meta.unit * kPD)[lane] =
                        make_float4(0.f, 0.f, 0.f, 0.f);
                    if (tid == 0) {
                        reinterpret_cast<PMeta*>(st + a.st_meta)->active = 0;
                        atomicOr(a.status, DAMP_EFLAG_NONFINITE);
                    }
                }
            }
        } else if (meta.unit >= 0 && warp == 0) {
            reinterpret_cast<float4*>(a.out + (size_t)meta.unit * kPD)[lane] =
                make_float4(0.f, 0.f, 0.f, 0.f);
            if (lane == 0 && meta.active < 0) atomicOr(a.status, DAMP_EFLAG_SLOT_RANGE);
        }

        // ---- step 2 (update) + step 6: X = S' + b delta^T, requantize in place
        if (any && !bad) {
            float am[kRW];
#pragma unroll
            for (int p = 0; p < kPP; ++p) {
                const float4 bs = tab->bs[p];
                const float2 bp = make_float2(bs.x, bs.y);
#pragma unroll
                for (int c = 0; c < 4; ++c) x[p][c] = __ffma2_rn(bp, dl[c], x[p][c]);
                am[2 * p] = __uint_as_float(__reduce_max_sync(
                    0xffffffffu, __float_as_uint(absmax4v(x[p][0].x, x[p][1].x, x[p][2].x, x[p][3].x))));
                am[2 * p + 1] = __uint_as_float(__reduce_max_sync(
                    0xffffffffu, __float_as_uint(absmax4v(x[p][0].y, x[p][1].y, x[p][2].y, x[p][3].y))));
            }
            if (lane == 0) {
#pragma unroll
                for (int i = 0; i < kRW; i += 4)
                    *reinterpret_cast<float4*>(&tab->amax[i]) = make_float4(am[i], am[i + 1], am[i + 2], am[i + 3]);
            }
            __syncwarp();
            // per byte row r = lane & 15: inv = fl(Q/a) into the table (lanes
            // 0-15), scale = fl(a/Q) into the block (lanes 16-31)
            {
                const int r = lane & 15;
                const bool byte_row = !((m16 >> r) & 1u);
                const float am_r = tab->amax[r];
                if constexpr (FP8) {
                    float res = 0.f;
                    if (byte_row) res = lane < 16 ? __fdiv_rn(kQ, am_r) : __fdiv_rn(am_r, kQ);
                    const float inv_r = __shfl_sync(0xffffffffu, res, r);
                    if (byte_row) {
                        const bool zero = am_r == 0.0f || isinf(inv_r);
                        if (lane < 16) tab->inv[r] = zero ? 0.0f : res;
                        else *reinterpret_cast<float*>(blk + tab->soff[r]) = zero ? 0.0f : res;
                    }
                } else {
                    // every lane forms both: inv by IEEE division, scale by
                    // division by the constant 127 (Markstein: one product and
                    // two fused corrections give the correctly rounded
                    // quotient for every finite a >= 0; a = inf is kept)
                    const float inv = __fdiv_rn(127.0f, am_r);
                    const float y = 0.007874015718698501587f;   // RN(1/127)
                    const float q0 = __fmul_rn(am_r, y);
                    const float q1 = __fmaf_rn(__fmaf_rn(-q0, 127.0f, am_r), y, q0);
                    const float scale = isinf(am_r) ? am_r : q1;
                    if (byte_row) {
                        const bool zero = am_r == 0.0f || isinf(inv);
                        if (lane < 16) tab->inv[r] = zero ? 0.0f : inv;
                        else *reinterpret_cast<float*>(blk + tab->soff[r]) = zero ? 0.0f : scale;
                    }
                }
            }
            __syncwarp();
#pragma unroll
            for (int p = 0; p < kPP; ++p) {
                const uint2 o = tab->off[p];
                const float2 ip = *reinterpret_cast<const float2*>(&tab->inv[2 * p]);
                if constexpr (ROWS == kRowsMixed) {
                    const uint2 cw = quant_pair4<false>(x[p], ip);
                    const uint32_t s4 = smem_u32(b4);
                    pair_store(p, m16, s4 + o.x, s4 + o.y, cw, x[p]);
                } else {
                    // INT8 or FP8 pools hold no FP16 rows: two code words
                    const uint2 cw = quant_pair4<FP8>(x[p], ip);
                    *reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(b4) + o.x) = cw.x;
                    *reinterpret_cast<uint32_t*>(const_cast<uint8_t*>(b4) + o.y) = cw.y;
                }
            }
            fence_proxy_async_smem();
        }
        if (++stage == NS) {
            stage = 0;
            parity ^= 1u;
        }
    }

    // The last completed item (it-1) is still to be written back.
    __syncthreads();
    if (aborted) {
        // loads still landing in this CTA's stages: the items after the last
        // one consumed that the refill warp issued (it .. issued-1)
        if (warp == kIssueWarp) {
            if (lane == 0) {
                atomicOr(a.status, DAMP_EFLAG_TIMEOUT);
                for (int jt = it; jt < issued; ++jt)
                    (void)mbar_wait_bounded(full_bar(jt % NS), static_cast<uint32_t>(jt / NS) & 1u,
                                            100000000ull);
            }
        }
    }
    if (warp == kStoreWarp && lane == 0) {
        if (it >= 1) store_item(it - 1);
        bulk_wait_all<0>();
    }
}

// Stage layout within `budget` bytes of shared memory; returns the number of
// stages that fit (0 when fewer than three do).
uint32_t unit_layout(StepArgs& a, bool kda, bool bf16, uint32_t budget) {
    const uint32_t elt = bf16 ? 2 : 4;
    auto up = [](uint32_t x, uint32_t m) { return (x + m - 1) / m * m; };
    // a block may be read up to 8 bytes per lane past a row: keep 256 bytes of
    // the stage after the largest block
    uint32_t off = a.block_stride;
    a.st_q = off;
    off = up(off + kPD * elt, 16);
    a.st_k = off;
    off = up(off + kPD * elt, 16);
    a.st_v = off;
    off = up(off + kPD * elt, 16);
    a.st_alpha = off;
    off += kda ? kPD * 4 : 0;
    a.st_mask = off;
    a.st_dir = off;
    off += kDirBytes;
    a.st_meta = off;
    off += sizeof(PMeta);
    a.stage_bytes = up(off, 128);
    const uint32_t scratch =
        up((4 * kNW * kPD + 2 * kPD) * 4 + kNW * (uint32_t)sizeof(RowTab), 128);
    uint32_t ns = (budget - scratch - 128) / a.stage_bytes;
    if (ns > 6) ns = 6;
    if (ns < 3) return 0;
    a.n_stages = (int)ns;
    a.scratch_off = ns * a.stage_bytes;
    a.bar_off = a.scratch_off + scratch;
    return ns;
}

// Shared memory of one CTA: 227 KB alone on an SM; two CTAs share the SM's
// 228 KB, less 1 KB reserved per CTA.
constexpr uint32_t kBudget1 = 227u * 1024u;
constexpr uint32_t kBudget2 = 228u * 1024u / 2 - 1024u;

template <bool KDA, bool BF16, int ROWS>
cudaError_t unit_attrs_t() {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(decode_unit_kernel<KDA, BF16, ROWS>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(decode_unit_kernel<KDA, BF16, ROWS>,
                                            cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    });
    return attr_err;
}

template <bool KDA, bool BF16, int ROWS>
cudaError_t launch_unit_t(const StepArgs& a0, cudaStream_t stream) {
    auto kern = decode_unit_kernel<KDA, BF16, ROWS>;
    const cudaError_t attr_err = unit_attrs_t<KDA, BF16, ROWS>();
    if (attr_err != cudaSuccess) return attr_err;
    StepArgs a = a0;
    int dev = 0, sms = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    // two CTAs per SM when 3 stages fit in half of it, else one CTA
    uint32_t ns = unit_layout(a, KDA, BF16, kBudget2);
    if (ns == 0) ns = unit_layout(a, KDA, BF16, kBudget1);
    if (ns == 0) return cudaErrorInvalidConfiguration;
    const size_t smem = a.bar_off + 8u * ns;
    int per_sm = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kPT, smem)) != cudaSuccess)
        return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int grid = std::min(a.n_items, sms * per_sm);
    if (grid <= 0) return cudaSuccess;
    // launched as a programmatic dependent of the previous kernel on the
    // stream (the kernel waits for it before touching shared data)
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(kPT);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, a);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

template <int ROWS>
cudaError_t prepare_rows() {
    cudaError_t e;
    if ((e = unit_attrs_t<false, false, ROWS>()) != cudaSuccess) return e;
    if ((e = unit_attrs_t<false, true, ROWS>()) != cudaSuccess) return e;
    if ((e = unit_attrs_t<true, false, ROWS>()) != cudaSuccess) return e;
    return unit_attrs_t<true, true, ROWS>();
}

cudaError_t prepare_decode_unit() {
    cudaError_t e;
    if ((e = prepare_rows<kRowsMixed>()) != cudaSuccess) return e;
    if ((e = prepare_rows<kRowsInt8>()) != cudaSuccess) return e;
    return prepare_rows<kRowsFp8>();
}

bool decode_unit_fits(const StepArgs& a, int in_dtype, int gate) {
    StepArgs b = a;
    return unit_layout(b, gate == DAMP_GATE_VECTOR, in_dtype == DAMP_DTYPE_BF16, kBudget1) != 0;
}

template <int ROWS>
cudaError_t launch_rows(const StepArgs& a, bool kda, bool bf, cudaStream_t stream) {
    if (kda) return bf ? launch_unit_t<true, true, ROWS>(a, stream) : launch_unit_t<true, false, ROWS>(a, stream);
    return bf ? launch_unit_t<false, true, ROWS>(a, stream) : launch_unit_t<false, false, ROWS>(a, stream);
}

cudaError_t launch_decode_unit(const StepArgs& a, int in_dtype, int gate, bool fp8,
                               cudaStream_t stream) {
    const bool kda = gate == DAMP_GATE_VECTOR, bf = in_dtype == DAMP_DTYPE_BF16;
    if (fp8) return launch_rows<kRowsFp8>(a, kda, bf, stream);
    if (a.format == DAMP_FMT_INT8_ROW) return launch_rows<kRowsInt8>(a, kda, bf, stream);
    return launch_rows<kRowsMixed>(a, kda, bf, stream);
}

}  // namespace damp
