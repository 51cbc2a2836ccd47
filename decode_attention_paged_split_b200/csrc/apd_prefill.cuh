// apd_prefill.cuh -- sm_100a kernel of multi-query (chunked prefill) attention
// over the paged bf16 KV cache.
//
// The operation comes from the AstrAI commit log of csrc/kernels/attn_paged_decode.cu:
// prefill kernels templated on the paged KV policy, the unified causal_offset
// (-1 = off, >= 0 = position of the first query) and 2-D [batch, kv_len] / 3-D
// [batch, q_len, kv_len] masks that may be combined with causal.  The B200
// design is our own:
//
//  * A CTA owns 128 query rows of one (sequence b, kv head): the rows are the
//    (query i, head-in-group hh) pairs of that kv head in query-major order,
//    row = i * g + hh, so the g heads that share the kv head and several
//    consecutive queries fill the tensor-core M side together and each K/V tile
//    is read once for all 128 rows.
//  * Warp 8 is the producer: it resolves the page of each 32-token tile (32
//    page-table entries per coalesced load) and its lane 0 issues the TMA tiled
//    loads of the K and V tiles into a STAGES-deep ring; "full" mbarriers count
//    the bytes, "empty" mbarriers count the 8 consumer warps that released a
//    stage.  Every wait is bounded.
//  * Warps 0-7 each own 16 rows: Q is loaded once from global straight into
//    mma A-fragments; per tile S = Q K^T and O += P V run on mma.sync m16n8k16
//    (bf16 in, fp32 accumulate) with the K/V tile read by ldmatrix from the
//    conflict-free staged layout; the online softmax is fp32 with exp2 and
//    handles rows that see no key of a tile (or none at all: output zeros).
//  * A tile's columns are visible to a row when t < seq_len, t <= causal_offset
//    + i (if causal) and the mask allows it; tiles past the block's last
//    visible key are not loaded.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "apd_kernels.cuh"
#include "apd_ptx.cuh"

namespace apd {

// Consumer warps per CTA: 8 (128 query rows) for D <= 128; 4 (64 rows) for D = 256,
// whose 128 fp32 accumulators per lane leave no registers for more warps.
template <int D>
struct PrefillShape {
    static constexpr int kConsumers = (D == 256) ? 4 : 8;
    static constexpr int kRows = 16 * kConsumers;
    static constexpr int kThreads = 32 * (kConsumers + 1);
};

struct PrefillParams {
    const __nv_bfloat16* q;   // [B, Lq, Hq, D]
    int64_t q_sb, q_si, q_sh;
    __nv_bfloat16* out;       // [B, Lq, Hq, D]
    int64_t o_sb, o_si, o_sh;
    const int32_t* page_table;
    int64_t pt_s0, pt_s1;
    const int32_t* seq_lens;
    const uint8_t* mask;      // NULL, [B, kv_len] or [B, Lq, kv_len]
    int64_t m_sb, m_si, m_st; // m_si = 0 for a 2-D mask
    uint32_t* flags;          // sticky device flags (may be NULL)
    int32_t B, Lq, Hq, Hkv, g, P, NP, MP;
    int32_t blocks_per_head;  // ceil(Lq * g / rows per CTA)
    int32_t causal_offset;
    float scale_log2;
};


template <int D, int STAGES>
__global__ void __launch_bounds__(PrefillShape<D>::kThreads, 1)
    prefill_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ CUtensorMap kmap,
                   const __grid_constant__ CUtensorMap vmap) {
    using G = Geometry<D>;
    constexpr int kPrefillConsumers = PrefillShape<D>::kConsumers;
    constexpr int kPrefillRows = PrefillShape<D>::kRows;
    constexpr uint32_t kStage = 2 * G::kKVTileBytes;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empty = full + STAGES;
    uint64_t* vzero = empty + STAGES;  // consumers meet here after zeroing the V tail (at most once)
    const uint32_t ring = (smem_u32(vzero + 1) + 1023u) & ~1023u;

    // ---- work item: (sequence b, kv head, block of kPrefillRows query rows)
    const int rb = blockIdx.x % p.blocks_per_head;
    const int bh = blockIdx.x / p.blocks_per_head;
    const int kvh = bh % p.Hkv;
    const int b = bh / p.Hkv;
    const int R = p.Lq * p.g;
    const int row0 = rb * kPrefillRows;

    if (threadIdx.x == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) {
            mbar_init(smem_u32(full + s), 1);
            mbar_init(smem_u32(empty + s), kPrefillConsumers);
        }
        {
            mbar_init(smem_u32(vzero), 32 * kPrefillConsumers);
        }
        fence_mbar_init();
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
    }
    // Launched with programmatic dependent launch: nothing above reads global
    // memory; from here on the previous kernel in the stream has finished.
    pdl_wait_prior_grid();

    const int64_t cap = static_cast<int64_t>(p.MP) * p.P;
    int L = __ldcg(p.seq_lens + b);
    if (L < 0 || L > cap) {
        if (p.flags && threadIdx.x == 0) atomicOr(p.flags, L < 0 ? kFlagLenNegative : kFlagLenClamped);
        L = L < 0 ? 0 : static_cast<int>(cap);
    }
    const int i_last = min(p.Lq - 1, (min(row0 + kPrefillRows, R) - 1) / p.g);
    int kv_end = L;  // keys this block can see: [0, kv_end)
    if (p.causal_offset >= 0) kv_end = max(0, min(L, p.causal_offset + i_last + 1));
    const int ntiles = (kv_end + kTile - 1) / kTile;
    __syncthreads();  // barriers initialised
    pdl_launch_dependents();

    if (warp == kPrefillConsumers) {
        // ---------------- producer warp
        const uint64_t pol = l2_policy_evict_last();  // other row blocks of this head read the same tiles
        int32_t pg = 0;
        for (int j = 0; j < ntiles; ++j) {
            if ((j & 31) == 0) {
                const int jj = j + lane;
                pg = 0;
                if (jj < ntiles) {
                    if (p.page_table == nullptr) {
                        pg = b;
                    } else {
                        const int pj = (jj * kTile) / p.P;
                        pg = __ldcg(p.page_table + static_cast<int64_t>(b) * p.pt_s0 + static_cast<int64_t>(pj) * p.pt_s1);
                    }
                }
            }
            const int32_t page = __shfl_sync(0xffffffffu, pg, j & 31);
            const int stage = j % STAGES;
            if (j >= STAGES &&
                !mbar_wait_bounded(smem_u32(empty + stage), static_cast<uint32_t>((j / STAGES) - 1) & 1u,
                                   kWaitTimeoutNs)) {
                if (lane == 0 && p.flags) atomicOr(p.flags, kFlagTimeout);
                return;
            }
            if (lane == 0) {
                if (page < 0 || page >= p.NP) {
                    if (p.flags) atomicOr(p.flags, kFlagPageOOR);
                }
                const uint32_t bar = smem_u32(full + stage);
                const uint32_t sbase = ring + static_cast<uint32_t>(stage) * kStage;
                const int slot = (j * kTile) % p.P;
                mbar_arrive_expect_tx(bar, kStage);
                if constexpr (D == 32) {
                    tma_load_4d(sbase, &kmap, bar, 0, kvh, slot, page, pol);
                    tma_load_4d(sbase + G::kKVTileBytes, &vmap, bar, 0, kvh, slot, page, pol);
                } else {
                    tma_load_5d(sbase, &kmap, bar, 0, kvh, slot, page, 0, pol);
                    tma_load_5d(sbase + G::kKVTileBytes, &vmap, bar, 0, kvh, slot, page, 0, pol);
                }
            }
            __syncwarp();
        }
        return;
    }

    // ---------------- consumer warps: 16 query rows each (rows gq and gq + 8 per lane)
    const int tq = lane & 3, gq = lane >> 2, mi = lane >> 3;
    const int r_lo = row0 + 16 * warp + gq, r_hi = r_lo + 8;
    const bool ok_lo = r_lo < R, ok_hi = r_hi < R;
    const int i_lo = ok_lo ? r_lo / p.g : 0, i_hi = ok_hi ? r_hi / p.g : 0;
    const int h_lo = kvh * p.g + (ok_lo ? r_lo - i_lo * p.g : 0);
    const int h_hi = kvh * p.g + (ok_hi ? r_hi - i_hi * p.g : 0);
    int lim_lo = ok_lo ? L : 0, lim_hi = ok_hi ? L : 0;  // a row sees keys t < lim (and the mask)
    if (p.causal_offset >= 0) {
        lim_lo = min(lim_lo, p.causal_offset + i_lo + 1);
        lim_hi = min(lim_hi, p.causal_offset + i_hi + 1);
    }
    const uint8_t* mrow_lo = p.mask ? p.mask + b * p.m_sb + static_cast<int64_t>(i_lo) * p.m_si : nullptr;
    const uint8_t* mrow_hi = p.mask ? p.mask + b * p.m_sb + static_cast<int64_t>(i_hi) * p.m_si : nullptr;

    // Q rows straight from global into the mma A-fragments
    uint32_t qf[G::kSteps][4];
    {
        const __nv_bfloat16* q_lo = p.q + b * p.q_sb + i_lo * p.q_si + h_lo * p.q_sh;
        const __nv_bfloat16* q_hi = p.q + b * p.q_sb + i_hi * p.q_si + h_hi * p.q_sh;
#pragma unroll
        for (int ks = 0; ks < G::kSteps; ++ks) {
            const int c0 = 16 * ks + 2 * tq;
            qf[ks][0] = ok_lo ? *reinterpret_cast<const uint32_t*>(q_lo + c0) : 0u;
            qf[ks][1] = ok_hi ? *reinterpret_cast<const uint32_t*>(q_hi + c0) : 0u;
            qf[ks][2] = ok_lo ? *reinterpret_cast<const uint32_t*>(q_lo + c0 + 8) : 0u;
            qf[ks][3] = ok_hi ? *reinterpret_cast<const uint32_t*>(q_hi + c0 + 8) : 0u;
        }
    }

    float acc[G::kNTiles][4];
#pragma unroll
    for (int nd = 0; nd < G::kNTiles; ++nd) acc[nd][0] = acc[nd][1] = acc[nd][2] = acc[nd][3] = 0.f;
    float m_lo = -INFINITY, m_hi = -INFINITY, l_lo = 0.f, l_hi = 0.f;

    for (int j = 0; j < ntiles; ++j) {
        const int stage = j % STAGES;
        if (!mbar_wait_bounded(smem_u32(full + stage), static_cast<uint32_t>(j / STAGES) & 1u, kWaitTimeoutNs)) {
            if (lane == 0 && p.flags) atomicOr(p.flags, kFlagTimeout);
            return;
        }
        const uint32_t sbase = ring + static_cast<uint32_t>(stage) * kStage;
        const uint32_t vb = sbase + G::kKVTileBytes;
        // V rows past the sequence end hold anything (NaN included): zero them before
        // any consumer multiplies them by a zero weight.
        const int valid = L - kTile * j;
        if (valid < kTile) {
            for (int idx = warp * 32 + lane; idx < (kTile - valid) * G::kChunks; idx += 32 * kPrefillConsumers) {
                st_shared_zero16(vb + G::chunk_off(valid + idx / G::kChunks, idx % G::kChunks, kTile));
            }
            // an mbarrier with a bounded wait rather than a named barrier: a consumer that
            // gave up on an earlier wait cannot leave the others blocked here
            mbar_arrive(smem_u32(vzero));
            if (!mbar_wait_bounded(smem_u32(vzero), 0u, kWaitTimeoutNs)) {
                if (lane == 0 && p.flags) atomicOr(p.flags, kFlagTimeout);
                return;
            }
        }

        // ---- S = Q K^T over the tile's 32 keys
        float s[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < G::kSteps; ++ks) {
#pragma unroll
            for (int np = 0; np < 2; ++np) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4(sbase + G::chunk_off(8 * (2 * np + (mi >> 1)) + (lane & 7), 2 * ks + (mi & 1), kTile), b0,
                        b1, b2, b3);
                mma_bf16_16816(s[2 * np], qf[ks], b0, b1);
                mma_bf16_16816(s[2 * np + 1], qf[ks], b2, b3);
            }
        }
        // ---- visibility: length, causal offset and mask, per row
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) {
            const int t0 = kTile * j + 8 * nt + 2 * tq;
            const bool v0 = t0 < lim_lo && (!mrow_lo || mrow_lo[t0 * p.m_st]);
            const bool v1 = t0 + 1 < lim_lo && (!mrow_lo || mrow_lo[(t0 + 1) * p.m_st]);
            const bool v2 = t0 < lim_hi && (!mrow_hi || mrow_hi[t0 * p.m_st]);
            const bool v3 = t0 + 1 < lim_hi && (!mrow_hi || mrow_hi[(t0 + 1) * p.m_st]);
            s[nt][0] = v0 ? s[nt][0] * p.scale_log2 : -INFINITY;
            s[nt][1] = v1 ? s[nt][1] * p.scale_log2 : -INFINITY;
            s[nt][2] = v2 ? s[nt][2] * p.scale_log2 : -INFINITY;
            s[nt][3] = v3 ? s[nt][3] * p.scale_log2 : -INFINITY;
        }

        // ---- online softmax; a row that has seen no key keeps m = -inf and takes
        // 0 as its reference so that exp2 gives exact zeros, never NaN
        float mx_lo = fmaxf(fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1])),
                            fmaxf(fmaxf(s[2][0], s[2][1]), fmaxf(s[3][0], s[3][1])));
        float mx_hi = fmaxf(fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3])),
                            fmaxf(fmaxf(s[2][2], s[2][3]), fmaxf(s[3][2], s[3][3])));
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
        const float mn_lo = fmaxf(m_lo, mx_lo), mn_hi = fmaxf(m_hi, mx_hi);
        const float ref_lo = (mn_lo == -INFINITY) ? 0.f : mn_lo;
        const float ref_hi = (mn_hi == -INFINITY) ? 0.f : mn_hi;
        const float alpha_lo = exp2f(m_lo - ref_lo), alpha_hi = exp2f(m_hi - ref_hi);
        m_lo = mn_lo;
        m_hi = mn_hi;
        uint32_t pa[2][4];
        float rs_lo = 0.f, rs_hi = 0.f;
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int nt = 2 * kk + h;
                const uint32_t plo = pack_bf16x2(exp2f(s[nt][0] - ref_lo), exp2f(s[nt][1] - ref_lo));
                const uint32_t phi = pack_bf16x2(exp2f(s[nt][2] - ref_hi), exp2f(s[nt][3] - ref_hi));
                pa[kk][2 * h] = plo;
                pa[kk][2 * h + 1] = phi;
                rs_lo += bf16_lo(plo) + bf16_hi(plo);
                rs_hi += bf16_lo(phi) + bf16_hi(phi);
            }
        }
        l_lo = l_lo * alpha_lo + rs_lo;
        l_hi = l_hi * alpha_hi + rs_hi;
#pragma unroll
        for (int nd = 0; nd < G::kNTiles; ++nd) {
            acc[nd][0] *= alpha_lo;
            acc[nd][1] *= alpha_lo;
            acc[nd][2] *= alpha_hi;
            acc[nd][3] *= alpha_hi;
        }
        // ---- O += P V
#pragma unroll
        for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
            for (int nd = 0; nd < G::kNTiles; nd += 2) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_trans(vb + G::chunk_off(16 * kk + 8 * (mi & 1) + (lane & 7), nd + (mi >> 1), kTile), b0, b1,
                              b2, b3);
                mma_bf16_16816(acc[nd], pa[kk], b0, b1);
                mma_bf16_16816(acc[nd + 1], pa[kk], b2, b3);
            }
        }
        // ---- release the stage to the producer (the tail zeroing, a generic-proxy
        // write, is ordered before the TMA refill of this stage)
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_u32(empty + stage));
    }

    // ---- epilogue: out = acc / l; a row that saw no key gets zeros
    float ll = l_lo + __shfl_xor_sync(0xffffffffu, l_lo, 1);
    ll += __shfl_xor_sync(0xffffffffu, ll, 2);
    float lh = l_hi + __shfl_xor_sync(0xffffffffu, l_hi, 1);
    lh += __shfl_xor_sync(0xffffffffu, lh, 2);
    const float il = ll > 0.f ? 1.f / ll : 0.f, ih = lh > 0.f ? 1.f / lh : 0.f;
    __nv_bfloat16* o_lo = p.out + b * p.o_sb + i_lo * p.o_si + h_lo * p.o_sh;
    __nv_bfloat16* o_hi = p.out + b * p.o_sb + i_hi * p.o_si + h_hi * p.o_sh;
#pragma unroll
    for (int nd = 0; nd < G::kNTiles; ++nd) {
        const int d = 8 * nd + 2 * tq;
        if (ok_lo) *reinterpret_cast<uint32_t*>(o_lo + d) = pack_bf16x2(acc[nd][0] * il, acc[nd][1] * il);
        if (ok_hi) *reinterpret_cast<uint32_t*>(o_hi + d) = pack_bf16x2(acc[nd][2] * ih, acc[nd][3] * ih);
    }
}

}  // namespace apd
