// damp_decode.cu -- the decode-step kernel of libdamp (sm_100a).
//
// One decode step of a DAMP-style compressed recurrent state for every
// (batch entry, head) unit ("DAMP: Decay-Aware Mixed-Precision Recurrent-State
// Quantization", both abstracts; step order of "STEPQuant ...", Appendix
// Table C2, steps 1, 2, 3 and 6):
//   reconstruct S^ (FP16 rows exact, INT8 rows code*scale)      step 1
//   S' = D S^, u = k^T S', X = S' + (beta k)(v - u)^T           step 2
//   out = X^T q, before requantization                          step 3
//   requantize X in place (FP16 rows, INT8 rows + FP32 scale)   step 6
//
// Work decomposition.  A persistent CTA of 8 warps walks work items (128/d
// units each) with a grid stride.  Each thread keeps a (d/8) x 4 tile of the
// state in registers from the dequantize through the requantize, so shared
// memory is read once and written once per unit.  Warp 7, idle while columns
// are combined, is also the issue warp: its lanes hold the next units'
// metadata (slot, gates); it moves later units' state blocks and inputs into
// free shared-memory stages with cp.async.bulk (no tensor map, no multicast),
// completing on the stage's mbarrier.  Thread 0 writes each item's blocks
// back with one bulk store each as soon as they are requantized; a stage is
// refilled only after its store has read it.
// The in-place update is safe because a unit's block has exactly one reader
// and one writer per call (Table C2 step 6: the old representation stays
// valid until its reader is done) -- slot indices within a call are distinct.
//
// Numerics.  u_j is summed in the recursive pairwise order over key rows:
// each thread sums its d/8 consecutive rows as a subtree, the 8 row-group
// sums are combined by the top three levels of the same tree.  Together with
// the explicit round-to-nearest intrinsics (and -fmad=false) this makes X,
// and so every stored code, FP16 value and scale, a deterministic function of
// the inputs.  The readout uses out_j = w_j + c*delta_j with
// w = S'^T q and c = q^T (beta k), which equals X^T q up to FP32 rounding.
#include <cuda_runtime.h>

#include <algorithm>
#include <mutex>

#include "damp.h"
#include "damp_device.cuh"

namespace damp {
namespace {

constexpr int kThreads = 256;

struct Meta {  // one per unit in a stage, written by the issuing thread
    int slot;
    float alpha;  // GDN scalar decay
    float beta;
    int exists;   // unit index < n*H
};

template <bool BF16>
__device__ __forceinline__ float load_in(const uint8_t* base, int idx) {
    if constexpr (BF16) {
        const uint16_t h = reinterpret_cast<const uint16_t*>(base)[idx];
        return __uint_as_float(static_cast<uint32_t>(h) << 16);
    } else {
        return reinterpret_cast<const float*>(base)[idx];
    }
}

// bf16 value i of a packed pair-of-bf16 word array
__device__ __forceinline__ float bf16_at(const uint32_t* w, int i) {
    return __uint_as_float((i & 1) ? (w[i >> 1] & 0xffff0000u) : (w[i >> 1] << 16));
}

template <int D, bool QUANT, bool KDA, bool BF16, bool FP8>
__global__ void __launch_bounds__(kThreads, 2) decode_step_kernel(const StepArgs a) {
    using G = Geo<D>;
    constexpr int RPT = G::RPT, UPI = G::UPI, LPR = G::LPR;
    constexpr int LOGR = (RPT == 2) ? 1 : (RPT == 4) ? 2 : (RPT == 8) ? 3 : 4;
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

    const int n_units = a.n * a.H;
    const int my_items = (a.n_items - (int)blockIdx.x + (int)gridDim.x - 1) / (int)gridDim.x;
    const int my_units = my_items * UPI;

    // ---- issue side (warp 0).  Lane L holds the metadata of CTA-local unit
    // U == L (mod 32), loaded 32 units ahead of use, so the slot lookups never
    // stall the pipeline.
    auto load_meta = [&](int U) {
        Meta m{-1, 0.f, 0.f, 0};
        if (U < my_units) {
            const int item = (int)blockIdx.x + (U / UPI) * (int)gridDim.x;
            const int u = item * UPI + U % UPI;
            if (u < n_units) {
                m.exists = 1;
                m.slot = __ldg(a.slot_idx + u / a.H);
                if constexpr (!KDA) m.alpha = __ldg(a.alpha + u);
                m.beta = __ldg(a.beta + u);
            }
        }
        return m;
    };
    constexpr int kIssueWarp = kThreads / 32 - 1;   // idle while columns are combined
    Meta ring{-1, 0.f, 0.f, 0};
    if (warp == kIssueWarp) ring = load_meta(lane);

    // Load work item `il` (CTA-local) into stage il % NS.  Issue warp only.
    auto issue = [&](int il) {
        const int stage = il % NS;
        uint8_t* st = smem + (size_t)stage * a.stage_bytes;
        const int src = (il * UPI + lane) & 31;          // lane holding unit (il, lane)
        Meta m;
        m.slot = __shfl_sync(0xffffffffu, ring.slot, src);
        m.alpha = __shfl_sync(0xffffffffu, ring.alpha, src);
        m.beta = __shfl_sync(0xffffffffu, ring.beta, src);
        m.exists = __shfl_sync(0xffffffffu, ring.exists, src);
        // refill the ring entries consumed by this item
        const int rel = (lane - il * UPI) & 31;
        if (rel < UPI) ring = load_meta(il * UPI + rel + 32);
        const bool load = lane < UPI && m.exists && m.slot >= 0 && m.slot < a.n_slots;
        const int item_l = (int)blockIdx.x + il * (int)gridDim.x;
        const int h_l = (item_l * UPI + lane) % a.H;
        // this head's block: offset inside the slot and size (heads may differ)
        const uint2 hb = load ? __ldg(reinterpret_cast<const uint2*>(a.heads + h_l)) : make_uint2(0u, 0u);
        uint32_t tx = 0;
        if (lane < UPI) {
            *reinterpret_cast<Meta*>(st + a.st_meta + lane * sizeof(Meta)) = m;
            if (load) tx = hb.y + 3u * D * ELT + (KDA ? 4u * D : 0u) + (QUANT ? 4u * D : 0u);
        }
        const uint32_t tx_all = __reduce_add_sync(0xffffffffu, tx);
        __syncwarp();
        const bool hold = il == 0 && (a.hooks & kHookHoldFirstItem);
        if (lane == 0 && !hold) {
            if (tx_all) mbar_arrive_expect_tx(full_bar(stage), tx_all);
            else mbar_arrive(full_bar(stage));
        }
        __syncwarp();
        if (load && !hold) {
            const int item = (int)blockIdx.x + il * (int)gridDim.x;
            const int u = item * UPI + lane;
            const int h = u % a.H;
            const uint32_t fb = full_bar(stage);
            bulk_g2s(smem_u32(st + lane * a.block_stride),
                     a.blocks + (size_t)m.slot * a.slot_stride + hb.x, hb.y, fb);
            const size_t io = (size_t)u * D * ELT;
            bulk_g2s(smem_u32(st + a.st_q + lane * D * ELT), static_cast<const uint8_t*>(a.q) + io,
                     D * ELT, fb);
            bulk_g2s(smem_u32(st + a.st_k + lane * D * ELT), static_cast<const uint8_t*>(a.k) + io,
                     D * ELT, fb);
            bulk_g2s(smem_u32(st + a.st_v + lane * D * ELT), static_cast<const uint8_t*>(a.v) + io,
                     D * ELT, fb);
            if constexpr (KDA)
                bulk_g2s(smem_u32(st + a.st_alpha + lane * D * 4), a.alpha + (size_t)u * D, D * 4,
                         fb);
            if constexpr (QUANT)
                bulk_g2s(smem_u32(st + a.st_dir + lane * D * 4), a.dir + (size_t)h * D, D * 4,
                         fb);
        }
    };

    // Stage of item il is refilled with item il + NS - 2 at the start of
    // iteration il + ... : items il .. il + NS - 2 are in flight while item il
    // is consumed; the stage of item il - 1 is still being stored.
    // One bulk store per loaded block of item j (thread 0).
    auto store_item = [&](int j) {
        const uint8_t* sj = smem + (size_t)(j % NS) * a.stage_bytes;
        const int item_j = (int)blockIdx.x + j * (int)gridDim.x;
#pragma unroll
        for (int w = 0; w < UPI; ++w) {
            const Meta m = *reinterpret_cast<const Meta*>(sj + a.st_meta + w * sizeof(Meta));
            if (m.exists && m.slot >= 0 && m.slot < a.n_slots) {
                const int uw = item_j * UPI + w;
                const uint2 hb = __ldg(reinterpret_cast<const uint2*>(a.heads + uw % a.H));
                bulk_s2g(a.blocks + (size_t)m.slot * a.slot_stride + hb.x,
                         smem_u32(sj + w * a.block_stride), hb.y);
            }
        }
        bulk_commit();
    };

    const int ahead = NS - 2;
    int issued = 0;   // items issued so far (meaningful in the issue warp)
    if (warp == kIssueWarp)
        for (; issued < ahead && issued < my_items; ++issued) issue(issued);

    // ---- consumer side (all 8 warps)
    const int ui = tid / G::TPU;        // unit within the item
    const int tu = tid % G::TPU;        // thread within the unit
    const int cg = tu % LPR;            // column group: columns 4cg..4cg+3
    const int rg = tu / LPR;            // row group: rows r0..r0+RPT-1
    const int r0 = rg * RPT;

    uint8_t* scratch = smem + a.scratch_off;
    float* red_u = reinterpret_cast<float*>(scratch);                  // [UPI][8][D]
    float* red_w = red_u + UPI * 8 * D;                                // [UPI][8][D]
    float* delta_s = red_w + UPI * 8 * D;                              // [UPI][D]
    float* cpart_s = delta_s + UPI * D;                                // [UPI][8]
    float* rowbuf = cpart_s + UPI * 8 + (ui * 8 + rg) * 2 * RPT;       // this row group's
    int* s_bad = reinterpret_cast<int*>(cpart_s + UPI * 8 + 16 * UPI * RPT);   // [UPI] (a.validate)

    int it = 0;
    bool aborted = false;
    for (; it < my_items; ++it) {
        const int item = (int)blockIdx.x + it * (int)gridDim.x;
        const int stage = it % NS;
        const uint32_t parity = static_cast<uint32_t>(it / NS) & 1u;
        // a warp whose wait gave up in any lane skips the item; the CTA leaves
        // the loop together at the first barrier below
        const bool ok =
            __all_sync(0xffffffffu, mbar_wait_bounded(full_bar(stage), parity, a.wait_ns));
        uint8_t* st = smem + (size_t)stage * a.stage_bytes;
        const Meta meta = *reinterpret_cast<const Meta*>(st + a.st_meta + ui * sizeof(Meta));
        if (tid < UPI) s_bad[tid] = 0;
        const int u = item * UPI + ui;
        const bool active = ok && meta.exists && meta.slot >= 0 && meta.slot < a.n_slots;
        uint8_t* blk = st + ui * a.block_stride;
        const uint8_t* sq = st + a.st_q + ui * D * ELT;
        const uint8_t* sk = st + a.st_k + ui * D * ELT;
        const float* salpha = reinterpret_cast<const float*>(st + a.st_alpha) + ui * D;

        float2 x[RPT][2];
        const uint32_t* sdir = reinterpret_cast<const uint32_t*>(st + a.st_dir) + ui * D;
        // k and q of this thread's rows (bf16 kept packed: two per word)
        uint32_t kw[BF16 ? RPT / 2 : 1], qw[BF16 ? RPT / 2 : 1];
        if (active) {
            if constexpr (BF16) {
#pragma unroll
                for (int i = 0; i < RPT / 2; ++i) {
                    kw[i] = reinterpret_cast<const uint32_t*>(sk)[r0 / 2 + i];
                    qw[i] = reinterpret_cast<const uint32_t*>(sq)[r0 / 2 + i];
                }
            }
            // ---- step 1: reconstruct S^
            if constexpr (QUANT) {
                load_tile_dir<D, FP8>(blk, sdir, r0, cg, x);
            } else {
#pragma unroll
                for (int i = 0; i < RPT; ++i) {
                    const float4 f = *reinterpret_cast<const float4*>(
                        blk + ((size_t)(r0 + i) * D + 4 * cg) * 4);
                    x[i][0] = make_float2(f.x, f.y);
                    x[i][1] = make_float2(f.z, f.w);
                }
            }
            // ---- step 2 (first half): S' = D S^; u = k^T S' (pairwise); w = q^T S'
            float2 stk[LOGR][2];
            float2 usum0 = f2(0.f), usum1 = f2(0.f);
            float2 w0 = f2(0.f), w1 = f2(0.f);
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const int r = r0 + i;
                const float al = KDA ? salpha[r] : meta.alpha;
                x[i][0] = __fmul2_rn(x[i][0], f2(al));
                x[i][1] = __fmul2_rn(x[i][1], f2(al));
                float kr, qr;
                if constexpr (BF16) {
                    kr = bf16_at(kw, i);
                    qr = bf16_at(qw, i);
                } else {
                    kr = load_in<false>(sk, r);
                    qr = load_in<false>(sq, r);
                }
                // leaf products rounded on their own (scalar multiplies: never
                // fused with the pairwise additions that follow)
                float2 v0 = mul2_rn(f2(kr), x[i][0]);
                float2 v1 = mul2_rn(f2(kr), x[i][1]);
#pragma unroll
                for (int b = 0; b < LOGR; ++b) {
                    if ((i >> b) & 1) {
                        v0 = __fadd2_rn(stk[b][0], v0);
                        v1 = __fadd2_rn(stk[b][1], v1);
                    } else {
                        stk[b][0] = v0;
                        stk[b][1] = v1;
                        break;
                    }
                }
                if (i == RPT - 1) {
                    usum0 = v0;
                    usum1 = v1;
                }
                w0 = __ffma2_rn(f2(qr), x[i][0], w0);
                w1 = __ffma2_rn(f2(qr), x[i][1], w1);
            }
            float* ru = red_u + (ui * 8 + rg) * D + 4 * cg;
            float* rw = red_w + (ui * 8 + rg) * D + 4 * cg;
            *reinterpret_cast<float4*>(ru) = make_float4(usum0.x, usum0.y, usum1.x, usum1.y);
            *reinterpret_cast<float4*>(rw) = make_float4(w0.x, w0.y, w1.x, w1.y);
            // c = q^T (beta k) over this row group: lane cg < RPT takes row r0 + cg
            float cp = 0.f;
            if (cg < RPT) {
                const float kr = load_in<BF16>(sk, r0 + cg), qr = load_in<BF16>(sq, r0 + cg);
                cp = __fmul_rn(qr, __fmul_rn(meta.beta, kr));
            }
#pragma unroll
            for (int off = LPR / 2; off >= 1; off >>= 1)
                cp += __shfl_xor_sync(0xffffffffu, cp, off);
            if (cg == 0) cpart_s[ui * 8 + rg] = cp;
        }
        // the store of item it-2 (committed by thread 0) must have read its
        // stage before the issue warp refills that stage below
        if (tid == 0 && it >= 2) bulk_wait_read<1>();
        if (bar_red_or(0, kThreads, ok ? 0 : 1)) {
            aborted = true;
            break;
        }
        if (warp == kIssueWarp && it + ahead < my_items) {
            issue(it + ahead);
            issued = it + ahead + 1;
        }

        // ---- step 2 (second half) + step 3: per column j, delta_j and out_j
        if (tu < D) {
            const int j = tu;
            if (active && a.validate) {
                const float aj = KDA ? salpha[j] : meta.alpha;
                if (!(isfinite(load_in<BF16>(sq, j)) && isfinite(load_in<BF16>(sk, j)) &&
                      isfinite(load_in<BF16>(st + a.st_v + ui * D * ELT, j)) && isfinite(aj) &&
                      isfinite(meta.beta)))
                    atomicOr(&s_bad[ui], 1);
            }
            if (active) {
                const float* cu = red_u + ui * 8 * D + j;
                const float* cw = red_w + ui * 8 * D + j;
                const float uj = __fadd_rn(__fadd_rn(__fadd_rn(cu[0 * D], cu[1 * D]),
                                                     __fadd_rn(cu[2 * D], cu[3 * D])),
                                           __fadd_rn(__fadd_rn(cu[4 * D], cu[5 * D]),
                                                     __fadd_rn(cu[6 * D], cu[7 * D])));
                float wj = 0.f, c = 0.f;
#pragma unroll
                for (int g = 0; g < 8; ++g) {
                    wj = __fadd_rn(wj, cw[g * D]);
                    c = __fadd_rn(c, cpart_s[ui * 8 + g]);
                }
                const float vj = load_in<BF16>(st + a.st_v + ui * D * ELT, j);
                const float dj = __fsub_rn(vj, uj);
                delta_s[ui * D + j] = dj;
                a.out[(size_t)u * D + j] = __fmaf_rn(c, dj, wj);
            } else if (meta.exists) {
                a.out[(size_t)u * D + j] = 0.f;
                if (j == 0 && meta.slot >= a.n_slots) atomicOr(a.status, DAMP_EFLAG_SLOT_RANGE);
            }
        }
        __syncthreads();
        if (active && s_bad[ui]) {
            // a non-finite input: the unit is skipped (out row zeroed, block
            // neither updated nor stored)
            if (tu < D) a.out[(size_t)u * D + tu] = 0.f;
            if (tu == 0) {
                reinterpret_cast<Meta*>(st + a.st_meta + ui * sizeof(Meta))->slot = -1;
                atomicOr(a.status, DAMP_EFLAG_NONFINITE);
            }
        }

        // ---- step 2 (update) + step 6: X = S' + b delta^T, requantize in place
        if (active && !s_bad[ui]) {
            const float4 dl = *reinterpret_cast<const float4*>(delta_s + ui * D + 4 * cg);
            const float2 d0 = make_float2(dl.x, dl.y), d1 = make_float2(dl.z, dl.w);
#pragma unroll
            for (int i = 0; i < RPT; ++i) {
                const float kr = BF16 ? bf16_at(kw, i) : load_in<BF16>(sk, r0 + i);
                const float b = __fmul_rn(meta.beta, kr);
                x[i][0] = __ffma2_rn(f2(b), d0, x[i][0]);
                x[i][1] = __ffma2_rn(f2(b), d1, x[i][1]);
            }
            if constexpr (QUANT) {
                store_tile_dir<D, FP8>(blk, sdir, r0, cg, x, rowbuf);
            } else {
#pragma unroll
                for (int i = 0; i < RPT; ++i)
                    *reinterpret_cast<float4*>(blk + ((size_t)(r0 + i) * D + 4 * cg) * 4) =
                        make_float4(x[i][0].x, x[i][0].y, x[i][1].x, x[i][1].y);
            }
            fence_proxy_async_smem();
        }
        __syncthreads();
        // ---- write back (one bulk store per block), right after the rows are
        // written: with one CTA of large (FP32) blocks per SM and three stages,
        // an earlier store frees the stage for the next load sooner
        if (tid == 0) store_item(it);
    }

    if (aborted && warp == kIssueWarp && lane == 0) {
        atomicOr(a.status, DAMP_EFLAG_TIMEOUT);
        // loads still landing in this CTA's stages: the items the issue warp
        // issued after the last one consumed (it .. issued-1)
        for (int jt = it; jt < issued; ++jt)
            (void)mbar_wait_bounded(full_bar(jt % NS), static_cast<uint32_t>(jt / NS) & 1u,
                                    100000000ull);
    }
    if (tid == 0) bulk_wait_all<0>();
}

// ---------------------------------------------------------------------- host

struct Layout {
    uint32_t stage_bytes, st_q, st_k, st_v, st_alpha, st_mask, st_dir, st_meta;
    uint32_t scratch_bytes;
};

inline uint32_t align_up(uint32_t x, uint32_t a) { return (x + a - 1) / a * a; }

Layout stage_layout(int d, uint32_t stride, int in_dtype, int gate) {
    const uint32_t upi = 128 / d, elt = (in_dtype == DAMP_DTYPE_BF16) ? 2 : 4;
    Layout L{};
    uint32_t off = upi * stride;
    L.st_q = off;
    off = align_up(off + upi * d * elt, 16);
    L.st_k = off;
    off = align_up(off + upi * d * elt, 16);
    L.st_v = off;
    off = align_up(off + upi * d * elt, 16);
    L.st_alpha = off;
    off += (gate == DAMP_GATE_VECTOR) ? upi * d * 4 : 0;
    L.st_mask = off;   // unused by the decode step (kept 0-sized)
    L.st_dir = off;
    off += upi * d * 4;
    L.st_meta = off;
    off += upi * sizeof(Meta);
    L.stage_bytes = align_up(off, 128);
    // red_u + red_w [128/d][8][d] each, delta [128], cpart [8*128/d], rowbuf 2*128,
    // non-finite flags [128/d]
    L.scratch_bytes = align_up((2 * 8 * 128 + 128 + 8 * upi + 2 * 128 + 8) * 4, 128);
    return L;
}

// Kernel attributes are set once per instantiation (at pool creation, so that a
// later launch can be captured into a CUDA graph with no set-up call inside).
template <int D, bool QUANT, bool KDA, bool BF16, bool FP8>
cudaError_t attrs_t() {
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    auto kern = decode_step_kernel<D, QUANT, KDA, BF16, FP8>;
    std::call_once(once, [&] {
        attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        227 * 1024);
        if (attr_err == cudaSuccess)
            attr_err = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                                            100);
    });
    return attr_err;
}

template <int D, bool QUANT, bool KDA, bool BF16, bool FP8>
cudaError_t launch_t(const StepArgs& a0, cudaStream_t stream) {
    auto kern = decode_step_kernel<D, QUANT, KDA, BF16, FP8>;
    const cudaError_t attr_err = attrs_t<D, QUANT, KDA, BF16, FP8>();
    if (attr_err != cudaSuccess) return attr_err;

    StepArgs a = a0;
    int dev = 0, sms = 0, smem_sm = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess)
        return e;
    if ((e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor,
                                    dev)) != cudaSuccess)
        return e;
    const Layout L = stage_layout(D, a.block_stride, BF16 ? DAMP_DTYPE_BF16 : DAMP_DTYPE_F32,
                                  KDA ? DAMP_GATE_VECTOR : DAMP_GATE_SCALAR);
    // Two CTAs per SM when at least three stages fit, else one CTA with as many
    // stages as fit (up to 8).
    const uint32_t per_cta_2 = static_cast<uint32_t>(smem_sm) / 2 - 1024;
    const uint32_t per_cta_1 = 227u * 1024u;
    auto stages_for = [&](uint32_t budget) {
        const uint32_t fixed = L.scratch_bytes + 128;
        if (budget <= fixed) return 0u;
        uint32_t ns = (budget - fixed) / L.stage_bytes;
        return ns > 8 ? 8u : ns;
    };
    uint32_t ns = stages_for(per_cta_2);
    if (ns < 3) ns = stages_for(per_cta_1);
    if (ns < 3) return cudaErrorInvalidConfiguration;
    a.n_stages = static_cast<int>(ns);
    a.stage_bytes = L.stage_bytes;
    a.st_q = L.st_q;
    a.st_k = L.st_k;
    a.st_v = L.st_v;
    a.st_alpha = L.st_alpha;
    a.st_mask = L.st_mask;
    a.st_dir = L.st_dir;
    a.st_meta = L.st_meta;
    a.scratch_off = ns * L.stage_bytes;
    a.bar_off = a.scratch_off + L.scratch_bytes;
    const size_t smem = a.bar_off + 8u * ns;
    int per_sm = 0;
    if ((e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, smem)) !=
        cudaSuccess)
        return e;
    if (per_sm < 1) return cudaErrorInvalidConfiguration;
    const int grid = std::min(a.n_items, sms * per_sm);
    kern<<<grid, kThreads, smem, stream>>>(a);
    return cudaGetLastError();
}

// Codec of the byte rows: 0 = FP32 state (no byte rows), 1 = INT8, 2 = FP8 E4M3.
template <int D, int CODEC>
cudaError_t dispatch_codec(const StepArgs& a, int in_dtype, int gate, cudaStream_t s) {
    constexpr bool Q = CODEC != 0, F8 = CODEC == 2;
    const bool kda = gate == DAMP_GATE_VECTOR, bf = in_dtype == DAMP_DTYPE_BF16;
    if (kda) return bf ? launch_t<D, Q, true, true, F8>(a, s) : launch_t<D, Q, true, false, F8>(a, s);
    return bf ? launch_t<D, Q, false, true, F8>(a, s) : launch_t<D, Q, false, false, F8>(a, s);
}

inline int codec_of(int format) {
    return format == DAMP_FMT_FP32 ? 0 : format == DAMP_FMT_FP8_ROW ? 2 : 1;
}

template <int D>
cudaError_t dispatch_fmt(const PoolDesc& p, const StepArgs& a, int in_dtype, int gate,
                         cudaStream_t s) {
    switch (codec_of(p.format)) {
        case 0: return dispatch_codec<D, 0>(a, in_dtype, gate, s);
        case 2: return dispatch_codec<D, 2>(a, in_dtype, gate, s);
        default: return dispatch_codec<D, 1>(a, in_dtype, gate, s);
    }
}

template <int D, int CODEC>
cudaError_t prepare_codec() {
    constexpr bool Q = CODEC != 0, F8 = CODEC == 2;
    cudaError_t e;
    if ((e = attrs_t<D, Q, false, false, F8>()) != cudaSuccess) return e;
    if ((e = attrs_t<D, Q, false, true, F8>()) != cudaSuccess) return e;
    if ((e = attrs_t<D, Q, true, false, F8>()) != cudaSuccess) return e;
    return attrs_t<D, Q, true, true, F8>();
}

template <int D>
cudaError_t prepare_d(int codec) {
    switch (codec) {
        case 0: return prepare_codec<D, 0>();
        case 2: return prepare_codec<D, 2>();
        default: return prepare_codec<D, 1>();
    }
}

}  // namespace

cudaError_t prepare_decode(const PoolDesc& p) {
    const int c = codec_of(p.format);
    cudaError_t e;
    if (p.d_k != p.d_v) return cudaSuccess;   // the one-CTA-per-unit kernel needs no set-up
    switch (p.d_k) {
        case 16: return prepare_d<16>(c);
        case 32: return prepare_d<32>(c);
        case 64: return prepare_d<64>(c);
        case 128:
            if ((e = prepare_d<128>(c)) != cudaSuccess) return e;
            return c != 0 ? prepare_decode_unit() : cudaSuccess;
        default: return cudaSuccess;
    }
}

// Kernel choice.  a.n_items counts units on entry.  d = 128 quantized states:
// the row-pair kernel (damp_decode_unit.cu) whenever three stages of a block
// fit in shared memory; square d in {16, 32, 64, 128}: the thread-tile kernel
// above (an item holds 128/d units); every other shape: the one-CTA-per-unit
// kernel (damp_decode_any.cu).
cudaError_t launch_decode_step(const PoolDesc& p, const StepArgs& a0, int in_dtype, int gate,
                               cudaStream_t stream) {
    StepArgs a = a0;
    if (p.d_k == 128 && p.d_v == 128 && codec_of(p.format) != 0 &&
        decode_unit_fits(a, in_dtype, gate))
        return launch_decode_unit(a, in_dtype, gate, codec_of(p.format) == 2, stream);
    if (p.d_k != p.d_v || p.d_k > kMaxFastD || (p.d_k & (p.d_k - 1)))
        return launch_decode_any(a, in_dtype, gate, stream);
    const int upi = kMaxFastD / p.d_k;
    a.n_items = (a.n_items + upi - 1) / upi;
    switch (p.d_k) {
        case 16: return dispatch_fmt<16>(p, a, in_dtype, gate, stream);
        case 32: return dispatch_fmt<32>(p, a, in_dtype, gate, stream);
        case 64: return dispatch_fmt<64>(p, a, in_dtype, gate, stream);
        case 128: return dispatch_fmt<128>(p, a, in_dtype, gate, stream);
        default: return cudaErrorInvalidValue;
    }
}

}  // namespace damp
