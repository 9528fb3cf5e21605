// damp_decode_unit.cu -- decode step for quantized d = 128 states, one unit
// (slot, head) per CTA iteration, two CTAs per SM.
//
// Same arithmetic, same order of operations and same results as the generic
// kernel in damp_decode.cu ("STEPQuant ...", Appendix Table C2 steps 1, 2,
// 3, 6 on the DAMP row format); only the work decomposition differs.
//
// CTA of 8 warps.  Half-warp k = 2w + hh of warp w owns key rows [8g, 8g + 8)
// of the unit, g = order[k] from the head's row-group order in the pool header;
// a lane owns 8 columns, so one row takes 16 lanes.  Each thread keeps its
// 8 x 8 tile in registers from dequantize to requantize, and the per-row work
// (directory lookup, scale, k/q values, row maximum, division, stores) is
// spread over 8 columns.  The two halves of a warp work on different rows, so
// a format branch runs both paths, each for its half, where the rows differ in
// format; the order pairs groups whose FP16 rows line up, so that this is
// rare.  u = k^T S' is summed in the recursive pairwise order: 8 rows per
// thread as a subtree, then the top four levels over the 16 row groups by
// group index, whichever half-warp computed them.
//
// Two CTAs share an SM whenever three stages fit in half of its shared
// memory (4 stages at 27 FP16 rows): their barriers are independent, so one CTA's arithmetic fills the
// other's barrier waits.  While columns are combined, warp 6 writes back the
// previous unit's block (one bulk store, once the barrier after phase A has
// ordered every writer's fenced rows before it) and warp 7 refills the
// pipeline (cp.async.bulk of the block, q, k, v, the KDA decays and the
// head's row directory into a shared-memory ring of stages completing on
// mbarriers; no tensor map, no multicast).  A named barrier between the two
// lets the refill start as soon as the stage's old store has read it.  An
// item needs two CTA barriers, not three.

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
constexpr int kPR = 8;         // rows per thread
constexpr int kPG = 16;        // row groups (half-warps)
constexpr uint32_t kDirBytes = kDirStride * 4;   // directory + row-group order

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

template <bool BF16>
__device__ __forceinline__ float in_at(const uint8_t* base, int idx) {
    if constexpr (BF16) {
        return __uint_as_float(static_cast<uint32_t>(reinterpret_cast<const uint16_t*>(base)[idx])
                               << 16);
    } else {
        return reinterpret_cast<const float*>(base)[idx];
    }
}

__device__ __forceinline__ float bf16w(const uint32_t* w, int i) {
    return __uint_as_float((i & 1) ? (w[i >> 1] & 0xffff0000u) : (w[i >> 1] << 16));
}

// 8 byte-row codes (two words) times the row scale: INT8 or FP8 E4M3 codes.
template <bool FP8>
__device__ __forceinline__ void dq_byte8(uint2 w, float s, float2 (&x)[4]) {
    if constexpr (FP8) {
        dequant_e4m3x4(w.x, s, x[0], x[1]);
        dequant_e4m3x4(w.y, s, x[2], x[3]);
    } else {
        dequant_int8x4_packed(w.x, s, x[0], x[1]);
        dequant_int8x4_packed(w.y, s, x[2], x[3]);
    }
}
__device__ __forceinline__ void dq_fp16x8(uint4 h, float2 (&x)[4]) {
    dequant_fp16x4(make_uint2(h.x, h.y), x[0], x[1]);
    dequant_fp16x4(make_uint2(h.z, h.w), x[2], x[3]);
}
__device__ __forceinline__ float absmax8(const float2 (&x)[4]) {
    float m0, m1;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(m0) : "f"(fabsf(x[0].x)), "f"(fabsf(x[0].y)), "f"(fabsf(x[1].x)));
    asm("max.f32 %0, %1, %2, %3;" : "=f"(m1) : "f"(fabsf(x[1].y)), "f"(fabsf(x[2].x)), "f"(fabsf(x[2].y)));
    float m;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(m) : "f"(m0), "f"(m1), "f"(fabsf(x[3].x)));
    return fmaxf(m, fabsf(x[3].y));
}

template <bool KDA, bool BF16, bool FP8>
__global__ void __launch_bounds__(kPT, 2) decode_unit_kernel(const StepArgs a) {
    constexpr uint32_t ELT = BF16 ? 2 : 4;
    extern __shared__ __align__(128) uint8_t smem[];
    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int NS = a.n_stages;
    const uint32_t bar0 = smem_u32(smem + a.bar_off);
    auto full_bar = [&](int s) { return bar0 + 8u * s; };

    if (tid == 0) {
        for (int s = 0; s < NS; ++s) mbar_init(full_bar(s), 1);
        fence_mbar_init();
    }
    __syncthreads();

    const int H = a.H;
    const int my_items = (a.n_items - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;

    // ---- refill side (warp 7): lane L holds the metadata of CTA-local unit
    // U == L (mod 32), loaded 32 units ahead of use.  The ring holds raw
    // values: nothing waits for the loads until the unit is issued, and no
    // branch depends on a freshly loaded slot index.
    constexpr int kIssueWarp = kPT / 32 - 1;    // refill
    constexpr int kStoreWarp = kIssueWarp - 1;  // write-back
    struct RMeta {
        int slot;          // slot index; INT_MIN: no such unit
        float alpha, beta;
        int unit;
        int head;
        uint2 hb;          // the head's {block offset in the slot, block size}
    };
    auto load_meta = [&](int U) {
        RMeta r{INT_MIN, 0.f, 0.f, -1, 0, make_uint2(0u, 0u)};
        if (U < my_items) {
            const int u = (int)blockIdx.x + U * (int)gridDim.x;   // unit b*H + h
            const int b = u / H, h = u - b * H;
            r.head = h;
            r.slot = __ldg(a.slot_idx + b);
            r.unit = u;
            if constexpr (!KDA) r.alpha = __ldg(a.alpha + u);
            r.beta = __ldg(a.beta + u);
            r.hb = __ldg(reinterpret_cast<const uint2*>(a.heads + h));
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

    // Refill the stage of item il: metadata, then one bulk copy per operand,
    // all completing on the stage's mbarrier (lane 0 issues them).
    auto issue = [&](int il) {
        const int stage = il % NS;
        uint8_t* st = smem + (size_t)stage * a.stage_bytes;
        const int src = il & 31;
        RMeta r;
        r.slot = __shfl_sync(0xffffffffu, ring.slot, src);
        r.alpha = __shfl_sync(0xffffffffu, ring.alpha, src);
        r.beta = __shfl_sync(0xffffffffu, ring.beta, src);
        r.unit = __shfl_sync(0xffffffffu, ring.unit, src);
        r.head = __shfl_sync(0xffffffffu, ring.head, src);
        r.hb.x = __shfl_sync(0xffffffffu, ring.hb.x, src);
        r.hb.y = __shfl_sync(0xffffffffu, ring.hb.y, src);
        const PMeta m = finish_meta(r);
        if (lane == src) ring = load_meta(il + 32);
        if (lane == 0) {
            *reinterpret_cast<PMeta*>(st + a.st_meta) = m;
            const uint32_t fb = full_bar(stage);
            if (m.active == 1) {
                mbar_arrive_expect_tx(fb, m.bytes + 3u * kPD * ELT + (KDA ? 4u * kPD : 0u) + kDirBytes);
                bulk_g2s(smem_u32(st), a.blocks + m.boff, m.bytes, fb);
                const size_t io = (size_t)m.unit * kPD * ELT;
                bulk_g2s(smem_u32(st + a.st_q), static_cast<const uint8_t*>(a.q) + io, kPD * ELT, fb);
                bulk_g2s(smem_u32(st + a.st_k), static_cast<const uint8_t*>(a.k) + io, kPD * ELT, fb);
                bulk_g2s(smem_u32(st + a.st_v), static_cast<const uint8_t*>(a.v) + io, kPD * ELT, fb);
                if constexpr (KDA)
                    bulk_g2s(smem_u32(st + a.st_alpha), a.alpha + (size_t)m.unit * kPD, kPD * 4, fb);
                bulk_g2s(smem_u32(st + a.st_dir), a.dir + (size_t)r.head * kDirStride, kDirBytes, fb);
            } else {
                mbar_arrive(fb);
            }
        }
        __syncwarp();
    };

    // One bulk store of item j's block (store warp, lane 0).
    auto store_item = [&](int j) {
        const uint8_t* sj = smem + (size_t)(j % NS) * a.stage_bytes;
        const PMeta m = *reinterpret_cast<const PMeta*>(sj + a.st_meta);
        if (m.active == 1) bulk_s2g(a.blocks + m.boff, smem_u32(sj), m.bytes);
        bulk_commit();
    };

    const int ahead = NS - 2;
    if (warp == kIssueWarp)
        for (int il = 0; il < ahead && il < my_items; ++il) issue(il);

    // ---- consumers: half-warp k = 2w + hh of warp w owns row group order[k] of
    // the unit's head
    const int hh = lane >> 4;
    const int cg = lane & 15;           // columns 8cg .. 8cg+7

    uint8_t* scratch = smem + a.scratch_off;
    float* red_u = reinterpret_cast<float*>(scratch);   // [16][128], by row group
    float* red_w = red_u + kPG * kPD;                   // [16][128], by row group
    float* delta_s = red_w + kPG * kPD;                 // [128]
    float* cpart_s = delta_s + kPD;                     // [16], by row group
    float* rowbuf = cpart_s + kPG + (warp * 2 + hh) * 16;   // this half-warp's 16 floats

    int it = 0, stage = 0;
    uint32_t parity = 0;
    bool aborted = false;
    for (; it < my_items; ++it) {
        const bool ok = mbar_wait_bounded(full_bar(stage), parity);
        uint8_t* st = smem + (size_t)stage * a.stage_bytes;
        const PMeta meta = *reinterpret_cast<const PMeta*>(st + a.st_meta);
        const bool any = ok && meta.active == 1;
        // row group of this half-warp (the order is loaded with the directory)
        const int rg = any ? (st[a.st_dir + kDirWords * 4 + warp * 2 + hh] & (kPG - 1)) : warp * 2 + hh;
        const int r0 = rg * kPR;            // rows r0 .. r0+7
        uint8_t* blk = st;
        const uint8_t* sq = st + a.st_q;
        const uint8_t* sk = st + a.st_k;
        const float* salpha = reinterpret_cast<const float*>(st + a.st_alpha);
        const uint32_t* sdir = reinterpret_cast<const uint32_t*>(st + a.st_dir) + r0;
        const uint8_t* b16 = blk + cg * 16;
        const uint8_t* b8 = blk + cg * 8;

        float2 x[kPR][4];
        uint32_t kw[BF16 ? kPR / 2 : 1], qw[BF16 ? kPR / 2 : 1];
        auto kval = [&](int i) { return BF16 ? bf16w(kw, i) : in_at<false>(sk, r0 + i); };
        auto qval = [&](int i) { return BF16 ? bf16w(qw, i) : in_at<false>(sq, r0 + i); };
        uint32_t dir[kPR];
        // `any` is uniform over the CTA: the directory (and so every row
        // offset) is valid only for a loaded unit.
        if (any) {
            if constexpr (BF16) {
                const uint4 kv = *reinterpret_cast<const uint4*>(sk + 2 * r0);
                const uint4 qv = *reinterpret_cast<const uint4*>(sq + 2 * r0);
                kw[0] = kv.x; kw[1] = kv.y; kw[2] = kv.z; kw[3] = kv.w;
                qw[0] = qv.x; qw[1] = qv.y; qw[2] = qv.z; qw[3] = qv.w;
            }
            {
                const uint4 d0 = reinterpret_cast<const uint4*>(sdir)[0];
                const uint4 d1 = reinterpret_cast<const uint4*>(sdir)[1];
                dir[0] = d0.x; dir[1] = d0.y; dir[2] = d0.z; dir[3] = d0.w;
                dir[4] = d1.x; dir[5] = d1.y; dir[6] = d1.z; dir[7] = d1.w;
            }
            // ---- step 1: reconstruct S^ (all candidate reads first, then decode)
#pragma unroll
            for (int i0 = 0; i0 < kPR; i0 += 4) {
                uint4 w16[4];
                uint2 w8[4];
                float sc[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const uint32_t e = dir[i0 + j], off = e & 0xffffu;
                    w16[j] = *reinterpret_cast<const uint4*>(b16 + off);
                    w8[j] = *reinterpret_cast<const uint2*>(b8 + off);
                    sc[j] = *reinterpret_cast<const float*>(blk + ((e >> 16) & 0x7fffu));
                }
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    if (dir[i0 + j] >> 31) dq_fp16x8(w16[j], x[i0 + j]);
                    else dq_byte8<FP8>(w8[j], sc[j], x[i0 + j]);
                }
            }
            // ---- step 2 (first half): S' = D S^; u = k^T S' (pairwise); w = q^T S'
            float2 stk[3][4];
            float2 us[4], ws[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) ws[c] = f2(0.f);
#pragma unroll
            for (int i = 0; i < kPR; ++i) {
                const float al = KDA ? salpha[r0 + i] : meta.alpha;
                const float kr = kval(i), qr = qval(i);
                float2 v[4];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    x[i][c] = __fmul2_rn(x[i][c], f2(al));
                    v[c] = mul2_rn(f2(kr), x[i][c]);      // scalar products: never fused
                    ws[c] = __ffma2_rn(f2(qr), x[i][c], ws[c]);
                }
#pragma unroll
                for (int lv = 0; lv < 3; ++lv) {
                    if ((i >> lv) & 1) {
#pragma unroll
                        for (int c = 0; c < 4; ++c) v[c] = __fadd2_rn(stk[lv][c], v[c]);
                    } else {
#pragma unroll
                        for (int c = 0; c < 4; ++c) stk[lv][c] = v[c];
                        break;
                    }
                }
                if (i == kPR - 1) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) us[c] = v[c];
                }
            }
            float* ru = red_u + rg * kPD + 8 * cg;
            float* rw = red_w + rg * kPD + 8 * cg;
            reinterpret_cast<float4*>(ru)[0] = make_float4(us[0].x, us[0].y, us[1].x, us[1].y);
            reinterpret_cast<float4*>(ru)[1] = make_float4(us[2].x, us[2].y, us[3].x, us[3].y);
            reinterpret_cast<float4*>(rw)[0] = make_float4(ws[0].x, ws[0].y, ws[1].x, ws[1].y);
            reinterpret_cast<float4*>(rw)[1] = make_float4(ws[2].x, ws[2].y, ws[3].x, ws[3].y);
            // c = q^T (beta k) over this row group: lane cg < 8 takes row r0 + cg
            float cp = 0.f;
            if (cg < kPR) cp = __fmul_rn(in_at<BF16>(sq, r0 + cg),
                                         __fmul_rn(meta.beta, in_at<BF16>(sk, r0 + cg)));
#pragma unroll
            for (int off = 8; off >= 1; off >>= 1) cp += __shfl_xor_sync(0xffffffffu, cp, off);
            if (cg == 0) cpart_s[rg] = cp;
        }
        if (bar_red_or(0, kPT, ok ? 0 : 1)) {
            aborted = true;
            break;
        }

        // ---- write back item it-1 (its requantized rows were fenced by their
        // writers before this barrier) and refill the stage of item it-2 once
        // that item's store has read it: the store warp checks the read,
        // releases the refill warp through named barrier 2, then stores.
        if (warp == kStoreWarp) {
            if (lane == 0) bulk_wait_read<0>();
            __syncwarp();
            asm volatile("bar.arrive 2, 64;" ::: "memory");
            if (lane == 0 && it >= 1) store_item(it - 1);
        } else if (warp == kIssueWarp) {
            asm volatile("bar.sync 2, 64;" ::: "memory");
            if (it + ahead < my_items) issue(it + ahead);
        }
        // ---- step 2 (second half) + step 3: delta_j and out_j, 128 columns
        if (tid < kPD) {
            const int j = tid;
            if (meta.active == 1) {
                const float* c0 = red_u + j;
                float t[8];
#pragma unroll
                for (int q2 = 0; q2 < 8; ++q2)
                    t[q2] = __fadd_rn(c0[(2 * q2) * kPD], c0[(2 * q2 + 1) * kPD]);
                const float uj = __fadd_rn(
                    __fadd_rn(__fadd_rn(t[0], t[1]), __fadd_rn(t[2], t[3])),
                    __fadd_rn(__fadd_rn(t[4], t[5]), __fadd_rn(t[6], t[7])));
                const float* w0 = red_w + j;
                float wj = 0.f;
#pragma unroll
                for (int q2 = 0; q2 < kPG; ++q2) wj = __fadd_rn(wj, w0[q2 * kPD]);
                const float4* cpp = reinterpret_cast<const float4*>(cpart_s);
                float c = 0.f;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) {
                    const float4 v4 = cpp[q4];
                    c += (v4.x + v4.y) + (v4.z + v4.w);
                }
                const float vj = in_at<BF16>(st + a.st_v, j);
                const float dj = __fsub_rn(vj, uj);
                delta_s[j] = dj;
                a.out[(size_t)meta.unit * kPD + j] = __fmaf_rn(c, dj, wj);
            } else if (meta.unit >= 0) {
                a.out[(size_t)meta.unit * kPD + j] = 0.f;
                if (j == 0 && meta.active < 0) atomicOr(a.status, DAMP_EFLAG_SLOT_RANGE);
            }
        }
        __syncthreads();

        // ---- step 2 (update) + step 6: X = S' + b delta^T, requantize in place
        if (any) {
            const float4* dp = reinterpret_cast<const float4*>(delta_s + 8 * cg);
            const float4 d0 = dp[0], d1 = dp[1];
            const float2 dl[4] = {make_float2(d0.x, d0.y), make_float2(d0.z, d0.w),
                                  make_float2(d1.x, d1.y), make_float2(d1.z, d1.w)};
            float amax[kPR];
#pragma unroll
            for (int i = 0; i < kPR; ++i) {
                const float b = __fmul_rn(meta.beta, kval(i));
#pragma unroll
                for (int c = 0; c < 4; ++c) x[i][c] = __ffma2_rn(f2(b), dl[c], x[i][c]);
                // row maxima of both half-warps with full-warp reductions (the
                // other half contributes 0, the smallest |x|)
                const uint32_t mb = __float_as_uint(absmax8(x[i]));
                const uint32_t m0 = __reduce_max_sync(0xffffffffu, hh ? 0u : mb);
                const uint32_t m1 = __reduce_max_sync(0xffffffffu, hh ? mb : 0u);
                amax[i] = __uint_as_float(hh ? m1 : m0);
            }
            if (cg == 0) {
                reinterpret_cast<float4*>(rowbuf)[0] = make_float4(amax[0], amax[1], amax[2], amax[3]);
                reinterpret_cast<float4*>(rowbuf)[1] = make_float4(amax[4], amax[5], amax[6], amax[7]);
            }
            __syncwarp();
            if (cg < kPR) {
                const uint32_t e = sdir[cg];
                if (!(e >> 31)) {
                    float scale, inv;
                    row_scale<FP8>(rowbuf[cg], scale, inv);
                    rowbuf[kPR + cg] = inv;
                    *reinterpret_cast<float*>(blk + ((e >> 16) & 0x7fffu)) = scale;
                }
            }
            __syncwarp();
            const float4 i0 = reinterpret_cast<const float4*>(rowbuf)[2];
            const float4 i1 = reinterpret_cast<const float4*>(rowbuf)[3];
            const float inv[kPR] = {i0.x, i0.y, i0.z, i0.w, i1.x, i1.y, i1.z, i1.w};
            {
                const uint4 d0 = reinterpret_cast<const uint4*>(sdir)[0];
                const uint4 d1 = reinterpret_cast<const uint4*>(sdir)[1];
                dir[0] = d0.x; dir[1] = d0.y; dir[2] = d0.z; dir[3] = d0.w;
                dir[4] = d1.x; dir[5] = d1.y; dir[6] = d1.z; dir[7] = d1.w;
            }
#pragma unroll
            for (int i = 0; i < kPR; ++i) {
                const uint32_t e = dir[i], off = e & 0xffffu;
                if (e >> 31) {
                    const uint2 h0 = quant_fp16x4(x[i][0], x[i][1]);
                    const uint2 h1 = quant_fp16x4(x[i][2], x[i][3]);
                    *reinterpret_cast<uint4*>(const_cast<uint8_t*>(b16) + off) =
                        make_uint4(h0.x, h0.y, h1.x, h1.y);
                } else {
                    *reinterpret_cast<uint2*>(const_cast<uint8_t*>(b8) + off) =
                        FP8 ? make_uint2(quant_e4m3x4(x[i][0], x[i][1], inv[i]),
                                         quant_e4m3x4(x[i][2], x[i][3], inv[i]))
                            : make_uint2(quant_int8x4(x[i][0], x[i][1], inv[i]),
                                         quant_int8x4(x[i][2], x[i][3], inv[i]));
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
    if (warp == kStoreWarp && lane == 0) {
        if (it >= 1) store_item(it - 1);
        if (aborted) {
            atomicOr(a.status, DAMP_EFLAG_TIMEOUT);
            // drain loads that may still be landing in this CTA's stages
            for (int j = 0; j <= ahead; ++j) {
                const int jt = it + j;
                if (jt >= my_items) break;
                (void)mbar_wait_bounded(full_bar(jt % NS), static_cast<uint32_t>(jt / NS) & 1u,
                                        100000000ull);
            }
        }
        bulk_wait_all<0>();
    }
}

// Stage layout within `budget` bytes of shared memory; returns the number of
// stages that fit (0 when fewer than three do).
uint32_t unit_layout(StepArgs& a, bool kda, bool bf16, uint32_t budget) {
    const uint32_t elt = bf16 ? 2 : 4;
    auto up = [](uint32_t x, uint32_t m) { return (x + m - 1) / m * m; };
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
    const uint32_t scratch = up((2 * kPG * kPD + kPD + kPG + kPG * 16) * 4, 128);
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

template <bool KDA, bool BF16, bool FP8>
cudaError_t unit_attrs_t() {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(decode_unit_kernel<KDA, BF16, FP8>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(decode_unit_kernel<KDA, BF16, FP8>,
                                            cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    });
    return attr_err;
}

template <bool KDA, bool BF16, bool FP8>
cudaError_t launch_unit_t(const StepArgs& a0, cudaStream_t stream) {
    auto kern = decode_unit_kernel<KDA, BF16, FP8>;
    const cudaError_t attr_err = unit_attrs_t<KDA, BF16, FP8>();
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
    kern<<<grid, kPT, smem, stream>>>(a);
    return cudaGetLastError();
}

}  // namespace

cudaError_t prepare_decode_unit() {
    cudaError_t e;
    if ((e = unit_attrs_t<false, false, false>()) != cudaSuccess) return e;
    if ((e = unit_attrs_t<false, true, false>()) != cudaSuccess) return e;
    if ((e = unit_attrs_t<true, false, false>()) != cudaSuccess) return e;
    if ((e = unit_attrs_t<true, true, false>()) != cudaSuccess) return e;
    if ((e = unit_attrs_t<false, false, true>()) != cudaSuccess) return e;
    if ((e = unit_attrs_t<false, true, true>()) != cudaSuccess) return e;
    if ((e = unit_attrs_t<true, false, true>()) != cudaSuccess) return e;
    return unit_attrs_t<true, true, true>();
}

bool decode_unit_fits(const StepArgs& a, int in_dtype, int gate) {
    StepArgs b = a;
    return unit_layout(b, gate == DAMP_GATE_VECTOR, in_dtype == DAMP_DTYPE_BF16, kBudget1) != 0;
}

cudaError_t launch_decode_unit(const StepArgs& a, int in_dtype, int gate, bool fp8,
                               cudaStream_t stream) {
    const bool kda = gate == DAMP_GATE_VECTOR, bf = in_dtype == DAMP_DTYPE_BF16;
    if (fp8) {
        if (kda)
            return bf ? launch_unit_t<true, true, true>(a, stream)
                      : launch_unit_t<true, false, true>(a, stream);
        return bf ? launch_unit_t<false, true, true>(a, stream)
                  : launch_unit_t<false, false, true>(a, stream);
    }
    if (kda) return bf ? launch_unit_t<true, true, false>(a, stream) : launch_unit_t<true, false, false>(a, stream);
    return bf ? launch_unit_t<false, true, false>(a, stream) : launch_unit_t<false, false, false>(a, stream);
}

}  // namespace damp
