// apd_gemv.cuh -- sm_100a kernels of the decode projection y = x W^T for a bf16
// linear layer at decode time (M = 1..8 rows of x, weights [N, K]).
//
// The operation and the pieces taken from the pages come from the AstrAI commit
// logs of astrai/extension/ops/gemv.py and docs/developer/decode_linear_benchmark.md:
// a bf16 GEMV for decode-time linear layers, M from 1 to 8, weights read with
// 128-bit accesses.  The B200 design is our own:
//
//  * The weight matrix is cut into work units of 16 rows x 256 columns (8 KB).
//    All units (m-tile major) are shared equally by the warps of a persistent
//    grid, so every warp streams the same number of bytes; a warp whose share
//    starts or ends inside an m-tile leaves an fp32 partial of that m-tile, and
//    a small sum kernel (PDL-launched) adds the partials of each such m-tile.
//    Adding them in the main kernel instead (the last warp to finish a tile,
//    found with an arrival counter) measured slower: the fences and atomics at
//    the end of each warp's share cost more than the second launch.
//  * Each warp runs its own ring of STAGES stages.  Lane 0 issues TMA tiled loads
//    (cp.async.bulk.tensor, 128-byte swizzle, bounds-filled with zeros past N and
//    K) of the W unit as 4 boxes of [16 rows][64]; completion by mbarrier bytes.
//  * x: when its M rows fit in shared memory beside the ring (XS), the CTA copies
//    them once, with rows padded to an odd number of 16-byte chunks so the 8-row
//    ldmatrix reads hit distinct banks; lanes whose x row is >= M or whose column
//    is >= K read a 16-byte zero chunk instead.  Otherwise each stage also loads
//    the unit's x columns as 4 TMA boxes of [8 rows][64] (rows >= M zero-filled),
//    which costs the TMA engine half again the W bytes.
//  * The product runs on tensor cores (mma.sync m16n8k16, bf16 in, fp32 accumulate)
//    with 16 W rows on M and the <= 8 rows of x on N.  At M = 8 a scalar FMA loop
//    would need about as many issue slots as the SMs have at full HBM bandwidth;
//    one mma per 512 bytes of W leaves the issue slots idle.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "apd_kernels.cuh"
#include "apd_ptx.cuh"

namespace apd {

constexpr int kGemvRows = 16;      // W rows per unit (mma M)
constexpr int kGemvCols = 256;     // W columns per unit
constexpr int kGemvXRows = 8;      // x rows staged per unit (mma N)
constexpr uint32_t kGemvWBytes = kGemvRows * kGemvCols * 2;   // 8 KB
constexpr uint32_t kGemvXBytes = kGemvXRows * kGemvCols * 2;  // 4 KB
constexpr uint32_t kGemvStageBytes = kGemvWBytes + kGemvXBytes;

struct GemvParams {
    const __nv_bfloat16* x;  // [M, K], row stride ldx (used when x is staged once per CTA)
    int64_t ldx;
    int32_t x_pitch;         // bytes per staged x row: 16 * (K / 8 | 1)
    __nv_bfloat16* y;
    int64_t y_sm, y_sn;  // element strides of y [M, N]
    float* part;         // [2 * workers][16][8] fp32 partials
    uint32_t* flags;
    int32_t M, N, K;
    int32_t mtiles;      // ceil(N / 16)
    int32_t ktiles;      // ceil(K / 256)
    int32_t num_workers, warps;
    int32_t cta_per_mtile;  // 1: CTA b owns m-tile b, its warps split the k-tiles and add their parts in shared memory
};

// Byte offset of 16-byte chunk `ch` (8 columns) of row `row` in a unit staged as
// 4 blocks of [rows][64] with the 128-byte swizzle (conflict-free for ldmatrix).
__device__ __forceinline__ uint32_t gemv_off(int row, int ch, int rows) {
    const uint32_t off = static_cast<uint32_t>((ch >> 3) * rows * 128 + row * 128 + (ch & 7) * 16);
    return off ^ (((off >> 7) & 7u) << 4);
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int c0, int c1,
                                            uint64_t pol) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "l"(pol)
        : "memory");
}

template <int STAGES, bool XS>
__global__ void __launch_bounds__(32 * 8, 1)
    gemv_kernel(const __grid_constant__ GemvParams p, const __grid_constant__ CUtensorMap wmap,
                const __grid_constant__ CUtensorMap xmap) {
    constexpr uint32_t kStage = XS ? kGemvWBytes : kGemvStageBytes;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int w = blockIdx.x * p.warps + warp;

    // shared memory: mbarriers | merge mbarrier | x rows (XS) | 16-byte zero chunk (XS) | stage ring
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    const uint32_t merge_bar = smem_u32(bars + p.warps * STAGES);
    const uint32_t xs = (merge_bar + 8u + 15u) & ~15u;
    const uint32_t xz = xs + (XS ? static_cast<uint32_t>(p.M * p.x_pitch) : 0u);
    const uint32_t ring = ((XS ? xz + 16u : xs) + 1023u) & ~1023u;
    if (threadIdx.x == 0) {
        prefetch_tensormap(&wmap);
        if (!XS) prefetch_tensormap(&xmap);
    }
    // x and W may be written by the previous kernel in the stream (PDL launch).
    pdl_wait_prior_grid();
    pdl_launch_dependents();

    const int64_t total = static_cast<int64_t>(p.mtiles) * p.ktiles;
    int64_t ws, we;
    int nparts = 1;  // CTA-per-m-tile mode: warps with k-tiles (those that add their parts)
    if (p.cta_per_mtile) {
        // m-tile blockIdx.x; warp `warp` takes k-tiles [warp K / W, (warp + 1) K / W)
        const int64_t t0 = static_cast<int64_t>(blockIdx.x) * p.ktiles;
        ws = t0 + (static_cast<int64_t>(warp) * p.ktiles) / p.warps;
        we = t0 + (static_cast<int64_t>(warp + 1) * p.ktiles) / p.warps;
        nparts = p.ktiles < p.warps ? p.ktiles : p.warps;
        if (threadIdx.x == 0) {
            mbar_init(merge_bar, static_cast<uint32_t>(32 * nparts));
            fence_mbar_init();
        }
        __syncthreads();
    } else {
        ws = w < p.num_workers ? static_cast<int64_t>((static_cast<uint64_t>(w) * total) / p.num_workers) : 0;
        we = w < p.num_workers ? static_cast<int64_t>((static_cast<uint64_t>(w + 1) * total) / p.num_workers) : 0;
    }
    const bool active = ws < we;

    const uint32_t bar0 = smem_u32(bars + warp * STAGES);
    const uint32_t wring = ring + static_cast<uint32_t>(warp) * STAGES * kStage;
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) mbar_init(bar0 + 8 * s, 1);
        fence_mbar_init();
    }
    __syncwarp();
    const uint64_t pol_stream = l2_policy_evict_first();
    const uint64_t pol_keep = l2_policy_evict_last();

    int64_t pi = ws;
    auto issue_next = [&](int stage) {
        if (pi >= we) return;
        const int mt = static_cast<int>(pi / p.ktiles);
        const int kt = static_cast<int>(pi - static_cast<int64_t>(mt) * p.ktiles);
        if (lane == 0) {
            const uint32_t bar = bar0 + 8 * stage;
            const uint32_t sbase = wring + static_cast<uint32_t>(stage) * kStage;
            mbar_arrive_expect_tx(bar, kStage);
#pragma unroll
            for (int kb = 0; kb < 4; ++kb) {
                const int k0 = kt * kGemvCols + 64 * kb;
                tma_load_2d(sbase + kb * kGemvRows * 128, &wmap, bar, k0, mt * kGemvRows, pol_stream);
                if (!XS) tma_load_2d(sbase + kGemvWBytes + kb * kGemvXRows * 128, &xmap, bar, k0, 0, pol_keep);
            }
        }
        ++pi;
    };
    // the first W loads go out before the CTA copies x, so the copy overlaps them
    if (active) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) issue_next(s);
    }
    if constexpr (XS) {
        // 8 loads in flight per thread before their stores (the store's memory clobber
        // would otherwise hold each load until the previous chunk is stored)
        const int kch = p.K / 8;
        constexpr int kBatch = 8;
        for (int idx0 = threadIdx.x; idx0 < p.M * kch; idx0 += kBatch * blockDim.x) {
            uint4 v[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int idx = idx0 + u * static_cast<int>(blockDim.x);
                const int r = idx / kch, c = idx - r * kch;
                if (idx < p.M * kch) v[u] = __ldg(reinterpret_cast<const uint4*>(p.x + r * p.ldx) + c);
            }
#pragma unroll
            for (int u = 0; u < kBatch; ++u) {
                const int idx = idx0 + u * static_cast<int>(blockDim.x);
                if (idx >= p.M * kch) break;
                const int r = idx / kch, c = idx - r * kch;
                asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(xs + static_cast<uint32_t>(r * p.x_pitch + 16 * c)),
                             "r"(v[u].x), "r"(v[u].y), "r"(v[u].z), "r"(v[u].w)
                             : "memory");
            }
        }
        if (threadIdx.x == 0) st_shared_zero16(xz);
        __syncthreads();
    }
    if (!active) return;

    const int tq = lane & 3, gq = lane >> 2, mi = lane >> 3;
    float acc[2][4];  // two accumulators per k-step parity, summed at the end
    int seg_start_kt = 0;    // k-tile where the current segment (one m-tile) began
    bool seg_first = true;   // the segment began at the start of this warp's share
    for (int64_t i = ws; i < we; ++i) {
        const int k = static_cast<int>(i - ws);
        const int stage = k % STAGES;
        const uint32_t parity = static_cast<uint32_t>(k / STAGES) & 1u;
        const int mt = static_cast<int>(i / p.ktiles);
        const int kt = static_cast<int>(i - static_cast<int64_t>(mt) * p.ktiles);
        if (kt == 0 || i == ws) {
            seg_start_kt = kt;
            seg_first = (i == ws);
#pragma unroll
            for (int h = 0; h < 2; ++h) acc[h][0] = acc[h][1] = acc[h][2] = acc[h][3] = 0.f;
        }
        if (!mbar_wait_bounded(bar0 + 8 * stage, parity, kWaitTimeoutNs)) {
            if (lane == 0) atomicOr(p.flags, kFlagTimeout);
            for (int s = 0; s < STAGES; ++s) {
                const int64_t t = i + s;
                if (t < pi) {
                    const int kk = static_cast<int>(t - ws);
                    mbar_wait_bounded(bar0 + 8 * (kk % STAGES), static_cast<uint32_t>(kk / STAGES) & 1u,
                                      kWaitTimeoutNs / 8);
                }
            }
            return;
        }
        const uint32_t sbase = wring + static_cast<uint32_t>(stage) * kStage;
        const uint32_t xbase = sbase + kGemvWBytes;
        // 16 k-steps of 16 columns: A = W rows (ldmatrix.x4), B = x rows (ldmatrix.x4 covers 2 k-steps)
#pragma unroll
        for (int ks2 = 0; ks2 < kGemvCols / 32; ++ks2) {
            uint32_t b[4];
            if constexpr (XS) {
                const int xr = lane & 7;
                const int kel = kt * kGemvCols + 8 * (4 * ks2 + mi);  // first column of this lane's chunk
                ldsm_x4((xr < p.M && kel < p.K) ? xs + static_cast<uint32_t>(xr * p.x_pitch + 2 * kel) : xz, b[0], b[1],
                        b[2], b[3]);
            } else {
                ldsm_x4(xbase + gemv_off(lane & 7, 4 * ks2 + mi, kGemvXRows), b[0], b[1], b[2], b[3]);
            }
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int ks = 2 * ks2 + h;
                uint32_t a[4];
                ldsm_x4(sbase + gemv_off((mi & 1) * 8 + (lane & 7), 2 * ks + (mi >> 1), kGemvRows), a[0], a[1], a[2],
                        a[3]);
                mma_bf16_16816(acc[h], a, b[2 * h], b[2 * h + 1]);
            }
        }
        fence_proxy_async_smem();
        __syncwarp();
        issue_next(stage);

        const bool seg_end = (kt == p.ktiles - 1) || (i == we - 1);
        if (seg_end) {
            float c[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) c[e] = acc[0][e] + acc[1][e];
            const int n_lo = mt * kGemvRows + gq, n_hi = n_lo + 8;
            const int m0 = 2 * tq, m1 = m0 + 1;
            // the segment covers the whole m-tile: it began at k-tile 0 and ends at the last one
            const bool full = (seg_start_kt == 0) && (kt == p.ktiles - 1);
            if (full) {
                if (n_lo < p.N) {
                    if (m0 < p.M) p.y[m0 * p.y_sm + n_lo * p.y_sn] = __float2bfloat16_rn(c[0]);
                    if (m1 < p.M) p.y[m1 * p.y_sm + n_lo * p.y_sn] = __float2bfloat16_rn(c[1]);
                }
                if (n_hi < p.N) {
                    if (m0 < p.M) p.y[m0 * p.y_sm + n_hi * p.y_sn] = __float2bfloat16_rn(c[2]);
                    if (m1 < p.M) p.y[m1 * p.y_sm + n_hi * p.y_sn] = __float2bfloat16_rn(c[3]);
                }
            } else if (p.cta_per_mtile) {
                // this warp's part of the m-tile, [16 rows][8 m] fp32, into its ring (idle now)
                float* dst = reinterpret_cast<float*>(smem + (wring - smem_u32(smem)));
                *reinterpret_cast<float2*>(dst + gq * kGemvXRows + m0) = make_float2(c[0], c[1]);
                *reinterpret_cast<float2*>(dst + (gq + 8) * kGemvXRows + m0) = make_float2(c[2], c[3]);
            } else {
                const int64_t slot = 2 * static_cast<int64_t>(w) + (seg_first ? 0 : 1);
                float* dst = p.part + slot * (kGemvRows * kGemvXRows);
                *reinterpret_cast<float2*>(dst + gq * kGemvXRows + m0) = make_float2(c[0], c[1]);
                *reinterpret_cast<float2*>(dst + (gq + 8) * kGemvXRows + m0) = make_float2(c[2], c[3]);
            }
            seg_first = false;
        }
    }
    if (p.cta_per_mtile && nparts >= 2) {
        // every lane's part is in shared memory: arrive; the last warp (never empty) waits,
        // bounded, for the other parts and writes the m-tile's rows of y
        mbar_arrive(merge_bar);
        if (warp != p.warps - 1) return;
        if (!mbar_wait_bounded(merge_bar, 0u, kWaitTimeoutNs)) {
            if (lane == 0) atomicOr(p.flags, kFlagTimeout);
            return;
        }
        float4 a = make_float4(0.f, 0.f, 0.f, 0.f);  // lane -> 4 of the m-tile's 128 (row, m) values
        for (int k = 0; k < p.warps; ++k) {
            if ((k * p.ktiles) / p.warps == ((k + 1) * p.ktiles) / p.warps) continue;  // no k-tiles: no part
            const float4 v = *reinterpret_cast<const float4*>(smem + (ring - smem_u32(smem)) +
                                                              static_cast<uint32_t>(k) * STAGES * kStage + 16 * lane);
            a.x += v.x;
            a.y += v.y;
            a.z += v.z;
            a.w += v.w;
        }
        const float av[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int idx = 4 * lane + e;
            const int row = idx / kGemvXRows, m = idx % kGemvXRows;
            const int n = static_cast<int>(blockIdx.x) * kGemvRows + row;
            if (n < p.N && m < p.M) p.y[m * p.y_sm + n * p.y_sn] = __float2bfloat16_rn(av[e]);
        }
    }
}

// One warp per m-tile: adds the fp32 partials of an m-tile that two or more
// warps shared and writes y.  m-tiles covered by one warp were written already.
// (One warp per worker boundary instead, 194 CTAs rather than 1,563 for lm_head,
// measured the same within 1 us: the CTAs of unsplit m-tiles exit at once.)
__global__ void __launch_bounds__(128) gemv_sum_kernel(const __grid_constant__ GemvParams p) {
    pdl_wait_prior_grid();
    pdl_launch_dependents();
    const int mt = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (mt >= p.mtiles) return;
    const int64_t total = static_cast<int64_t>(p.mtiles) * p.ktiles;
    const int64_t t0 = static_cast<int64_t>(mt) * p.ktiles;
    const int w_first = worker_of(t0, total, p.num_workers);
    const int w_last = worker_of(t0 + p.ktiles - 1, total, p.num_workers);
    if (w_first == w_last) return;
    // lane -> 4 of the tile's 128 (row, m) values
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    for (int wk = w_first; wk <= w_last; ++wk) {
        const int64_t a = run_start(wk, total, p.num_workers);
        if (a == run_start(wk + 1, total, p.num_workers)) continue;  // empty share: wrote nothing
        const int64_t slot = 2 * static_cast<int64_t>(wk) + ((wk == w_first && a != t0) ? 1 : 0);
        const float4 v = *(reinterpret_cast<const float4*>(p.part + slot * (kGemvRows * kGemvXRows)) + lane);
        s[0] += v.x;
        s[1] += v.y;
        s[2] += v.z;
        s[3] += v.w;
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        const int idx = 4 * lane + e;
        const int row = idx / kGemvXRows, m = idx % kGemvXRows;
        const int n = mt * kGemvRows + row;
        if (n < p.N && m < p.M) p.y[m * p.y_sm + n * p.y_sn] = __float2bfloat16_rn(s[e]);
    }
}


}  // namespace apd
