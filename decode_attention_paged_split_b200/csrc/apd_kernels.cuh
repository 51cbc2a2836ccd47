// apd_kernels.cuh -- sm_100a kernels of paged split-KV decode attention.
//
// The operation, and the pieces of the design taken from the pages, come from
// the AstrAI commit log of csrc/kernels/attn_paged_decode.cu: decode attention
// over a paged KV cache, head packing of the query heads that share a kv head
// onto tensor-core tiles, one page-table lookup per 32-token tile (a tile never
// straddles a page because page_size is a multiple of 32), split-KV partials
// o_part / ml_part, and a single combine kernel.  The B200 design around them is
// our own:
//
//  * The unit of work is a 32-token tile of one (sequence b, kv head, head
//    block).  All tiles of all units are laid out in one flattened index space
//    (b-major, then kv head / head block, then tile), found on the device from
//    a prefix sum of the per-sequence tile counts.
//  * split_kernel (auto splits, num_splits == 0): every warp is an independent
//    worker that owns a contiguous run of that space, an equal share of it, one per
//    resident warp of a persistent, SM-count-sized grid.  A warp that covers a
//    whole unit writes the final bf16 output; otherwise it writes an unnormalised
//    fp32 partial plus (m, l), and the combine kernel merges the partials of each
//    unit.
//  * unit_kernel: one CTA per unit when every unit gets an SM of its own (auto
//    splits with host-known lengths), or one CTA per split of a unit with fixed
//    splits (num_splits == k, the k page-aligned chunks of each unit).  The CTA's
//    warps claim its tiles one at a time and merge their parts in shared memory.
//  * Each warp runs its own STAGES-deep ring in shared memory.  Lane 0 issues
//    TMA tiled loads (cp.async.bulk.tensor, 128-byte swizzle) of the K and V
//    tiles [32 tokens x D] of the next tiles straight from the paged cache
//    (stored as D/64 blocks of [32 tokens][64], conflict-free for ldmatrix),
//    plus the unit's query rows when a unit starts; completion is tracked by
//    mbarrier transaction bytes.  Page-table entries are fetched 32 tiles ahead,
//    one coalesced load per warp.  Page indices outside the pool read as zeros
//    (TMA bounds fill) instead of faulting.
//  * QK^T and PV run on tensor cores (mma.sync m16n8k16, bf16 in, fp32
//    accumulate) with the g query heads of a kv head on the M side (padded to
//    16), so K/V are read once per kv head.  The softmax is the online form in
//    fp32 with exp2 (logits pre-multiplied by scale * log2 e) and quad shuffles.
//  * g > 16 takes ceil(g / 16) head blocks, one warp each.  In balanced mode they
//    share one K/V ring in their CTA (SHARE): the first fills it, the others
//    release each stage on an mbarrier, and every K/V tile leaves HBM once.
//  * LEAN selects the trimmed per-tile code: row sums from an mma against ones,
//    2^x from the SFU, no masking on full tiles, and no rescale while no row's
//    max grows.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "apd_ptx.cuh"

namespace apd {

constexpr int kTile = 32;          // tokens per tile (= rows of one TMA box)
constexpr int kMaxRows = 16;       // query heads per unit (mma M)
constexpr int kMaxWarps = 8;       // warps per CTA, upper bound (D >= 128, shared K/V rings)
// Warps per CTA, upper bound of the split kernel.  Small tiles leave a warp latency-bound,
// and their register footprint leaves room for more warps: 12 at D = 32 and 10 at D = 64
// with one ring per warp (the launch bound caps registers at 170 and 204).
template <int D, bool SHARE>
constexpr int kMaxWarpsD = SHARE ? kMaxWarps : (D == 32 ? 16 : (D == 64 ? 10 : kMaxWarps));
constexpr uint32_t kFlagPageOOR = 0x1u;
constexpr uint32_t kFlagLenClamped = 0x2u;
constexpr uint32_t kFlagLenNegative = 0x4u;
constexpr uint32_t kFlagTimeout = 0x8u;
constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // 2 s per async-copy wait

// Wait, as one warp, for phase `parity` of an mbarrier.  Every lane polls, and lane 0
// decides for the whole warp when to give up, so the lanes never part ways: once
// `abort_word` (if given) has been raised by another warp of the CTA, or after about
// timeout_ns, when lane 0 raises `abort_word` and sets kFlagTimeout in `flags` (each if
// given).  Returns false when it gave up.
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                          volatile uint32_t* abort_word, uint32_t* flags) {
    bool done = mbar_try_wait(bar, parity);
    if (__all_sync(0xffffffffu, done)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (!done) done = mbar_try_wait(bar, parity);
        if (__all_sync(0xffffffffu, done)) return true;
        if ((it & 15u) == 0) {
            int give_up = 0;
            if ((threadIdx.x & 31) == 0) {
                if (abort_word && *abort_word) give_up = 1;
                else if (global_timer_ns() - t0 > timeout_ns) give_up = 2;
            }
            give_up = __shfl_sync(0xffffffffu, give_up, 0);
            if (give_up) {
                if (give_up == 2 && (threadIdx.x & 31) == 0) {
                    if (abort_word) *abort_word = 1u;
                    if (flags) atomicOr(flags, kFlagTimeout);
                }
                return false;
            }
        }
    }
}

struct SplitParams {
    const int32_t* page_table;  // NULL: contiguous KV, sequence b is page b
    int64_t pt_s0, pt_s1;
    const int32_t* seq_lens;
    __nv_bfloat16* out;
    int64_t out_sb, out_sh;
    float* o_part;      // [slots][rows_max][D]
    float* ml_part;     // [slots][rows_max][2]
    int32_t* cum_out;   // [B + 1] prefix sum of tiles per sequence (for the combine)
    int32_t zero_empty;  // balanced mode with no combine kernel: write the rows of empty sequences
    uint32_t* flags;
    int32_t B, Hq, Hkv, g, HB, rows_max, P, NP, MP;
    int32_t mode;       // 0 balanced (split_kernel); 1 fixed splits, 2 one CTA per unit (unit_kernel)
    int32_t ksplit;     // fixed splits: k
    int32_t num_workers;
    int32_t groups;     // balanced mode: worker groups (num_workers = groups * Hkv * HB)
    int32_t warps;      // warps per CTA
    uint32_t stage_bytes, q_box_bytes;
    float scale_log2;
    uint64_t wait_ns;           // limit of each mbarrier wait (kWaitTimeoutNs; shorter in the self-test)
    int32_t test_skip_release;  // self-test only: followers never release a shared stage (0 otherwise)
};

struct CombineParams {
    const int32_t* cum;       // [B + 1] (written by the split kernel; unused by the combine itself)
    const int32_t* seq_lens;  // [B]: the combine recomputes its prefix sums from these
    int32_t MP, P;            // page-table capacity MP * P, for the same clamp as the split kernel
    const float* o_part;
    const float* ml_part;
    __nv_bfloat16* out;
    int64_t out_sb, out_sh;
    int32_t B, Hkv, g, HB, rows_max;
    int32_t mode, ksplit, num_workers, groups;
};

template <int D>
struct Geometry {
    static_assert(D == 32 || D == 64 || D == 128 || D == 256, "head_dim");
    static constexpr int kSteps = D / 16;              // k-steps of QK^T
    static constexpr int kNTiles = D / 8;              // 8-wide n-tiles of PV
    static constexpr int kChunks = D / 8;              // 16-byte chunks per row
    static constexpr uint32_t kKVTileBytes = kTile * D * 2;
    // TMA swizzle applied to a byte offset from a 1024-aligned base:
    // 128B mode XORs address bits [4:6] with [7:9]; 64B mode bits [4:5] with [7:8].
    __device__ __forceinline__ static uint32_t swz(uint32_t off) {
        if constexpr (D == 32) {
            return off ^ (((off >> 7) & 3u) << 4);
        } else {
            return off ^ (((off >> 7) & 7u) << 4);
        }
    }
    // Byte offset of 16-byte chunk `ch` (8 elements of the head dim) of row `row`
    // in a staged tile of `rows` rows.  D >= 64: the tile is stored as D/64 blocks
    // of [rows][64 elements], so each 128-byte swizzle row is one token (or query
    // head) and the 8 rows an ldmatrix reads fall in 8 distinct swizzle phases
    // (no bank conflicts).  D == 32: [rows][32 elements] with the 64-byte swizzle.
    __device__ __forceinline__ static uint32_t chunk_off(int row, int ch, int rows) {
        if constexpr (D == 32) {
            return swz(static_cast<uint32_t>(row * 64 + ch * 16));
        } else {
            return swz(static_cast<uint32_t>((ch >> 3) * rows * 128 + row * 128 + (ch & 7) * 16));
        }
    }
};

// Equal shares of [0, total) among `parts`: part w owns [run_start(w), run_start(w + 1)).
__device__ __forceinline__ int64_t run_start(int w, int64_t total, int parts) {
    return static_cast<int64_t>((static_cast<uint64_t>(w) * static_cast<uint64_t>(total)) / parts);
}

// The part whose share contains position i.
__device__ __forceinline__ int worker_of(int64_t i, int64_t total, int parts) {
    return static_cast<int>((static_cast<uint64_t>(i + 1) * static_cast<uint64_t>(parts) - 1) /
                            static_cast<uint64_t>(total));
}

// Largest b in [0, B) with cum[b] <= x (cum non-decreasing, cum[0] = 0).
__device__ __forceinline__ int find_seq(const int32_t* cum, int B, int x) {
    int lo = 0, hi = B - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (cum[mid] <= x) lo = mid;
        else hi = mid - 1;
    }
    return lo;
}

// Position s of the sequence-tile space (s = cum[b] + j, all sequences' tiles in
// sequence order) -> (sequence b, tile j, tiles of that sequence n).
__device__ __forceinline__ void decode_pos(int s, const int32_t* cum, int B, int& b, int& j, int& n) {
    b = find_seq(cum, B, s);
    n = cum[b + 1] - cum[b];
    j = s - cum[b];
}

// Step a cursor to the next position; only called when that position exists.
__device__ __forceinline__ void advance_pos(const int32_t* cum, int& b, int& j, int& n) {
    if (++j == n) {
        j = 0;
        do {
            ++b;
            n = cum[b + 1] - cum[b];
        } while (n == 0);
    }
}

// Page of the tile at position s (0 past `end`).
__device__ __forceinline__ int32_t fetch_page(const SplitParams& p, const int32_t* cum, int s, int end) {
    if (s >= end) return 0;
    int b, j, n;
    decode_pos(s, cum, p.B, b, j, n);
    if (p.page_table == nullptr) return b;  // contiguous KV: sequence b is "page" b of Lmax tokens
    const int pj = (j * kTile) / p.P;
    return __ldcg(p.page_table + static_cast<int64_t>(b) * p.pt_s0 + static_cast<int64_t>(pj) * p.pt_s1);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

template <int D>
__device__ __forceinline__ void write_zero_rows(const SplitParams& p, int b, int head0, int rows, int lane) {
    for (int idx = lane; idx < rows * (D / 2); idx += 32) {
        const int r = idx / (D / 2), d2 = idx % (D / 2);
        *reinterpret_cast<uint32_t*>(p.out + b * p.out_sb + (head0 + r) * p.out_sh + 2 * d2) = 0u;
    }
}

// The running state of one warp over the tiles of one unit: the query rows' mma A-fragments,
// the fp32 accumulators of O (rows gq and gq + 8 of the 16-row head tile, columns 8 nd +
// 2 tq, + 1), the row sums and the row maxima (in log2 units).  step() consumes one staged
// 32-token K/V tile.
template <int D, bool LEAN>
struct TileAcc {
    using G = Geometry<D>;
    uint32_t qf[G::kSteps][4];
    float acc[G::kNTiles][4];
    float accl[4];  // row sums: rows gq in [0], [1] and gq + 8 in [2], [3]
    float m_lo, m_hi;

    __device__ __forceinline__ void reset() {
        m_lo = m_hi = -INFINITY;
        accl[0] = accl[1] = accl[2] = accl[3] = 0.f;
#pragma unroll
        for (int nd = 0; nd < G::kNTiles; ++nd) acc[nd][0] = acc[nd][1] = acc[nd][2] = acc[nd][3] = 0.f;
    }

    // Q A-fragments from a staged [rows_max x D] tile: matrix m of ldmatrix.x4 = (rows
    // 8*(m&1).., k chunk m>>1); rows at and past `rows` are zero.
    __device__ __forceinline__ void load_q(uint32_t qbase, int rows_max, int rows, int lane) {
        const int gq = lane >> 2;
        const int mi = lane >> 3;
        int qrow = (mi & 1) * 8 + (lane & 7);
        if (qrow >= rows_max) qrow = 0;  // stay inside the loaded box
#pragma unroll
        for (int ks = 0; ks < G::kSteps; ++ks) {
            const uint32_t ch = 2 * ks + (mi >> 1);
            ldsm_x4(qbase + G::chunk_off(qrow, ch, rows_max), qf[ks][0], qf[ks][1], qf[ks][2], qf[ks][3]);
            if (gq >= rows) qf[ks][0] = qf[ks][2] = 0u;
            if (gq + 8 >= rows) qf[ks][1] = qf[ks][3] = 0u;
        }
    }

    // One tile at `sbase` ([K | V], each 32 tokens x D): S = Q K^T, tokens at and past `valid`
    // masked (and their V rows zeroed, so that 0 * (stale or NaN) never reaches the
    // accumulator), online softmax in log2 units, O += P V.
    __device__ __forceinline__ void step(uint32_t sbase, int valid, float scale_log2, int lane) {
        const int tq = lane & 3;   // thread in quad: token / d pair
        const int gq = lane >> 2;  // quad index: row within the 8-row half
        constexpr uint32_t kOnesBf16x2 = 0x3F803F80u;
        constexpr bool kLean = LEAN;
        (void)gq;

        // ---- S = Q K^T over the 32 tokens of the tile: 4 n-tiles of 8 tokens
        float s[4][4];
#pragma unroll
        for (int nt = 0; nt < 4; ++nt) s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
        {
            const int mi = lane >> 3;
#pragma unroll
            for (int ks = 0; ks < G::kSteps; ++ks) {
#pragma unroll
                for (int np = 0; np < 2; ++np) {
                    const int row = 8 * (2 * np + (mi >> 1)) + (lane & 7);
                    const uint32_t ch = 2 * ks + (mi & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(sbase + G::chunk_off(row, ch, kTile), b0, b1, b2, b3);
                    mma_bf16_16816(s[2 * np], qf[ks], b0, b1);
                    mma_bf16_16816(s[2 * np + 1], qf[ks], b2, b3);
                }
            }
        }

        // ---- mask tokens past the sequence end; zero their V rows
        auto mask_and_scale = [&]() {
#pragma unroll
            for (int nt = 0; nt < 4; ++nt) {
                const int t0 = 8 * nt + 2 * tq;
                s[nt][0] = (t0 < valid) ? s[nt][0] * scale_log2 : -INFINITY;
                s[nt][1] = (t0 + 1 < valid) ? s[nt][1] * scale_log2 : -INFINITY;
                s[nt][2] = (t0 < valid) ? s[nt][2] * scale_log2 : -INFINITY;
                s[nt][3] = (t0 + 1 < valid) ? s[nt][3] * scale_log2 : -INFINITY;
            }
        };
        if (valid < kTile) {
            const uint32_t vb = sbase + G::kKVTileBytes;
            for (int idx = lane; idx < (kTile - valid) * G::kChunks; idx += 32) {
                const int r = valid + idx / G::kChunks;
                const int ch = idx % G::kChunks;
                st_shared_zero16(vb + G::chunk_off(r, ch, kTile));
            }
            __syncwarp();
            if constexpr (kLean) mask_and_scale();
        } else if constexpr (kLean) {
            // a full tile: no token to mask
#pragma unroll
            for (int nt = 0; nt < 4; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) s[nt][e] *= scale_log2;
        }
        if constexpr (!kLean) mask_and_scale();

        // ---- online softmax (rows gq and gq + 8 of the head tile)
        float mx_lo = fmaxf(fmaxf(s[0][0], s[0][1]), fmaxf(s[1][0], s[1][1]));
        mx_lo = fmaxf(mx_lo, fmaxf(fmaxf(s[2][0], s[2][1]), fmaxf(s[3][0], s[3][1])));
        float mx_hi = fmaxf(fmaxf(s[0][2], s[0][3]), fmaxf(s[1][2], s[1][3]));
        mx_hi = fmaxf(mx_hi, fmaxf(fmaxf(s[2][2], s[2][3]), fmaxf(s[3][2], s[3][3])));
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 1));
        mx_lo = fmaxf(mx_lo, __shfl_xor_sync(0xffffffffu, mx_lo, 2));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 1));
        mx_hi = fmaxf(mx_hi, __shfl_xor_sync(0xffffffffu, mx_hi, 2));
        const float mn_lo = fmaxf(m_lo, mx_lo);  // finite: every tile has >= 1 valid token
        const float mn_hi = fmaxf(m_hi, mx_hi);
        uint32_t pa[2][4];
        if constexpr (kLean) {
            // Rescale only when some row's running max grew.  Otherwise alpha would be
            // 2^0 = 1 exactly, so skipping is exact, and after a sequence's first tiles the
            // maxima rarely move.
            if (__any_sync(0xffffffffu, (mn_lo != m_lo) || (mn_hi != m_hi))) {
                const float alpha_lo = ex2_approx(m_lo - mn_lo);  // 0 on the unit's first tile
                const float alpha_hi = ex2_approx(m_hi - mn_hi);
                m_lo = mn_lo;
                m_hi = mn_hi;
                accl[0] *= alpha_lo;
                accl[1] *= alpha_lo;
                accl[2] *= alpha_hi;
                accl[3] *= alpha_hi;
#pragma unroll
                for (int nd = 0; nd < G::kNTiles; ++nd) {
                    acc[nd][0] *= alpha_lo;
                    acc[nd][1] *= alpha_lo;
                    acc[nd][2] *= alpha_hi;
                    acc[nd][3] *= alpha_hi;
                }
            }
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int nt = 2 * kk + h;
                    pa[kk][2 * h + 0] = pack_bf16x2(ex2_approx(s[nt][0] - mn_lo), ex2_approx(s[nt][1] - mn_lo));
                    pa[kk][2 * h + 1] = pack_bf16x2(ex2_approx(s[nt][2] - mn_hi), ex2_approx(s[nt][3] - mn_hi));
                }
                // the normaliser sums exactly the bf16 weights that enter PV
                mma_bf16_16816(accl, pa[kk], kOnesBf16x2, kOnesBf16x2);
            }
        } else {
            const float alpha_lo = exp2f(m_lo - mn_lo);
            const float alpha_hi = exp2f(m_hi - mn_hi);
            m_lo = mn_lo;
            m_hi = mn_hi;
            float rs_lo = 0.f, rs_hi = 0.f;
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
                for (int h = 0; h < 2; ++h) {
                    const int nt = 2 * kk + h;
                    const uint32_t plo = pack_bf16x2(exp2f(s[nt][0] - mn_lo), exp2f(s[nt][1] - mn_lo));
                    const uint32_t phi = pack_bf16x2(exp2f(s[nt][2] - mn_hi), exp2f(s[nt][3] - mn_hi));
                    pa[kk][2 * h + 0] = plo;
                    pa[kk][2 * h + 1] = phi;
                    // the normaliser sums exactly the bf16 weights that enter PV
                    rs_lo += bf16_lo(plo) + bf16_hi(plo);
                    rs_hi += bf16_lo(phi) + bf16_hi(phi);
                }
            }
            accl[0] = accl[0] * alpha_lo + rs_lo;
            accl[2] = accl[2] * alpha_hi + rs_hi;
#pragma unroll
            for (int nd = 0; nd < G::kNTiles; ++nd) {
                acc[nd][0] *= alpha_lo;
                acc[nd][1] *= alpha_lo;
                acc[nd][2] *= alpha_hi;
                acc[nd][3] *= alpha_hi;
            }
        }

        // ---- O += P V: k = 32 tokens (2 steps), n = D (8-wide tiles)
        {
            const uint32_t vb = sbase + G::kKVTileBytes;
            const int mi = lane >> 3;
#pragma unroll
            for (int kk = 0; kk < 2; ++kk) {
#pragma unroll
                for (int nd = 0; nd < G::kNTiles; nd += 2) {
                    const int row = 16 * kk + 8 * (mi & 1) + (lane & 7);
                    const uint32_t ch = nd + (mi >> 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_trans(vb + G::chunk_off(row, ch, kTile), b0, b1, b2, b3);
                    mma_bf16_16816(acc[nd], pa[kk], b0, b1);
                    mma_bf16_16816(acc[nd + 1], pa[kk], b2, b3);
                }
            }
        }
    }

    // The rows' sums of weights (rows gq and gq + 8), complete in every lane of the quad.
    __device__ __forceinline__ void row_sums(float& ll, float& lh) const {
        ll = accl[0];
        lh = accl[2];
        if constexpr (!LEAN) {
            ll += __shfl_xor_sync(0xffffffffu, ll, 1);
            ll += __shfl_xor_sync(0xffffffffu, ll, 2);
            lh += __shfl_xor_sync(0xffffffffu, lh, 1);
            lh += __shfl_xor_sync(0xffffffffu, lh, 2);
        }
    }

    // out rows (normalised, bf16): row r of the head tile at o_row0 + r * out_sh.
    __device__ __forceinline__ void write_out(__nv_bfloat16* o_row0, int64_t out_sh, int rows, int lane) const {
        const int tq = lane & 3, gq = lane >> 2;
        float ll, lh;
        row_sums(ll, lh);
        const float il = 1.f / ll, ih = 1.f / lh;
        __nv_bfloat16* o_lo = o_row0 + gq * out_sh;
        __nv_bfloat16* o_hi = o_lo + 8 * out_sh;
#pragma unroll
        for (int nd = 0; nd < G::kNTiles; ++nd) {
            const int d = 8 * nd + 2 * tq;
            if (gq < rows) *reinterpret_cast<uint32_t*>(o_lo + d) = pack_bf16x2(acc[nd][0] * il, acc[nd][1] * il);
            if (gq + 8 < rows) *reinterpret_cast<uint32_t*>(o_hi + d) = pack_bf16x2(acc[nd][2] * ih, acc[nd][3] * ih);
        }
    }

    // An unnormalised part: accumulator rows at op + r * ost (fp32) and (m, l) pairs at mp + 2 r.
    __device__ __forceinline__ void write_part(float* op, int ost, float* mp, int rows, int lane) const {
        const int tq = lane & 3, gq = lane >> 2;
        float ll, lh;
        row_sums(ll, lh);
#pragma unroll
        for (int nd = 0; nd < G::kNTiles; ++nd) {
            const int d = 8 * nd + 2 * tq;
            if (gq < rows) *reinterpret_cast<float2*>(op + gq * ost + d) = make_float2(acc[nd][0], acc[nd][1]);
            if (gq + 8 < rows)
                *reinterpret_cast<float2*>(op + (gq + 8) * ost + d) = make_float2(acc[nd][2], acc[nd][3]);
        }
        if (tq == 0) {
            if (gq < rows) *reinterpret_cast<float2*>(mp + 2 * gq) = make_float2(m_lo, ll);
            if (gq + 8 < rows) *reinterpret_cast<float2*>(mp + 2 * (gq + 8)) = make_float2(m_hi, lh);
        }
    }
};

// Row stride (floats) of a unit part's accumulator rows in shared memory: 8 floats of
// padding put the 8 rows one warp store touches on different banks.
template <int D>
constexpr int kPartStride = D + 8;

// Merge of the parts of one unit in unit_kernel: part k's (m, l) rows at ml_k = the start of
// warp k's first ring stage, its accumulator rows [kMaxRows][kPartStride] (fp32) 128
// bytes later.
// Warp `part` of `nparts` merges rows part, part + nparts, ...:
//   M = max_k m_k over parts with l_k > 0, out = sum_k 2^(m_k - M) acc_k / sum_k 2^(m_k - M) l_k.
// With `slot` >= 0 the merged part is written unnormalised to partial slot `slot` instead (the
// accumulator sum_k 2^(m_k - M) acc_k and (M, sum_k 2^(m_k - M) l_k)), for the combine kernel.
template <int D>
__device__ __noinline__ void unit_merge(const SplitParams& p, const uint8_t* ring0, uint32_t warp_bytes,
                                        int b, int head0, int rows, int part, int nparts, int lane, int64_t slot) {
    constexpr int kVec = D / 32;  // consecutive columns per lane
    for (int r = part; r < rows; r += nparts) {
        float M = -INFINITY;
        for (int k = 0; k < nparts; ++k) {
            const float* ml = reinterpret_cast<const float*>(ring0 + static_cast<size_t>(k) * warp_bytes);
            if (ml[2 * r + 1] > 0.f) M = fmaxf(M, ml[2 * r]);
        }
        float den = 0.f, acc[kVec];
#pragma unroll
        for (int e = 0; e < kVec; ++e) acc[e] = 0.f;
        for (int k = 0; k < nparts; ++k) {
            const float* ml = reinterpret_cast<const float*>(ring0 + static_cast<size_t>(k) * warp_bytes);
            if (!(ml[2 * r + 1] > 0.f)) continue;
            const float wk = exp2f(ml[2 * r] - M);
            den += wk * ml[2 * r + 1];
            const float* a = ml + 2 * kMaxRows + r * kPartStride<D> + kVec * lane;
            float v[kVec];  // this lane's kVec consecutive columns, in 16- (or 8-) byte loads
            if constexpr (kVec % 4 == 0) {
#pragma unroll
                for (int e = 0; e < kVec; e += 4) *reinterpret_cast<float4*>(v + e) = *reinterpret_cast<const float4*>(a + e);
            } else if constexpr (kVec == 2) {
                *reinterpret_cast<float2*>(v) = *reinterpret_cast<const float2*>(a);
            } else {
                v[0] = a[0];
            }
#pragma unroll
            for (int e = 0; e < kVec; ++e) acc[e] += wk * v[e];
        }
        if (slot >= 0) {
            float* po = p.o_part + (slot * p.rows_max + r) * D + kVec * lane;
#pragma unroll
            for (int e = 0; e < kVec; ++e) po[e] = acc[e];
            if (lane == 0) *reinterpret_cast<float2*>(p.ml_part + (slot * p.rows_max + r) * 2) = make_float2(M, den);
            continue;
        }
        const float inv = den > 0.f ? 1.f / den : 0.f;
        __nv_bfloat16* o = p.out + b * p.out_sb + (head0 + r) * p.out_sh + kVec * lane;
        if constexpr (kVec == 1) {
            o[0] = __float2bfloat16_rn(acc[0] * inv);
        } else {
#pragma unroll
            for (int e = 0; e < kVec; e += 2)
                *reinterpret_cast<uint32_t*>(o + e) = pack_bf16x2(acc[e] * inv, acc[e + 1] * inv);
        }
    }
}

// SHARE (balanced mode with g > 16, so HB = ceil(g / 16) head blocks per kv head): the HB
// warps of one kv head, which walk the same positions in one CTA, share one K/V ring, which
// the first of them (the leader) fills.  Before refilling a stage the leader waits on that
// stage's `empty` mbarrier, on which the other HB - 1 warps arrive once they have read the
// tile.  Each warp loads its own Q rows into a Q ring of its own.  Shared-memory layout:
// [K/V rings, one per kv head of the CTA][Q rings, one per warp], so a CTA of HB warps
// holds one K/V ring instead of HB.
template <int D, int STAGES, bool SHARE, bool LEAN>
__global__ void __launch_bounds__(32 * kMaxWarpsD<D, SHARE>, 1)
    split_kernel(const __grid_constant__ SplitParams p, const __grid_constant__ CUtensorMap kmap,
                 const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap qmap) {
    using G = Geometry<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int B = p.B;

    // ---- shared-memory carve-up: mbarriers, lengths, prefix sums, stage ring
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    uint64_t* empties = bars + p.warps * STAGES;  // SHARE: stage released by the followers
    // raised by a warp that gave up on a wait: the CTA's other waits then give up too
    volatile uint32_t* s_abort = reinterpret_cast<volatile uint32_t*>(empties + (SHARE ? p.warps * STAGES : 0));
    int32_t* s_len = reinterpret_cast<int32_t*>(empties + (SHARE ? p.warps * STAGES : 0) + 1);
    int32_t* s_cum = s_len + B;
    const uint32_t meta_end = smem_u32(s_cum + B + 1);
    const uint32_t ring = (meta_end + 1023u) & ~1023u;

    if (tid == 0) {
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
        prefetch_tensormap(&qmap);
    }
    // Launched with programmatic dependent launch: this CTA may start while the
    // previous kernel in the stream is still running.  Nothing above touches
    // global memory; from here on, that kernel has finished and its writes are
    // visible.
    pdl_wait_prior_grid();

    // ---- per-sequence tile counts and their prefix sum (every CTA, from L2)
    const int64_t cap = static_cast<int64_t>(p.MP) * p.P;
    uint32_t len_flags = 0;
    for (int b = tid; b < B; b += blockDim.x) {
        int L = __ldcg(p.seq_lens + b);
        if (L < 0) {
            L = 0;
            len_flags |= kFlagLenNegative;
        }
        if (L > cap) {
            L = static_cast<int>(cap);
            len_flags |= kFlagLenClamped;
        }
        s_len[b] = L;
        s_cum[b + 1] = (L + kTile - 1) / kTile;
    }
    if (tid == 0) {
        s_cum[0] = 0;
        *s_abort = 0u;
    }
    if (len_flags && blockIdx.x == 0) atomicOr(p.flags, len_flags);
    __syncthreads();
    if (SHARE && warp == 1) {
        // every warp's ring barriers, before any warp waits on another warp's
        for (int i = lane; i < p.warps * STAGES; i += 32) {
            mbar_init(smem_u32(bars + i), 1);
            mbar_init(smem_u32(empties + i), static_cast<uint32_t>(p.HB - 1));
        }
        fence_mbar_init();
    }
    if (warp == 0) {
        const int per = (B + 31) / 32;
        const int lo = 1 + lane * per;
        const int hi = min(lo + per, B + 1);
        int sum = 0;
        for (int i = lo; i < hi; ++i) sum += s_cum[i];
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        int run = incl - sum;
        for (int i = lo; i < hi; ++i) {
            run += s_cum[i];
            s_cum[i] = run;
        }
    }
    __syncthreads();
    if (blockIdx.x == 0) {
        for (int i = tid; i <= B; i += blockDim.x) p.cum_out[i] = s_cum[i];
    }
    // The combine kernel may start its launch now; it waits (griddepcontrol.wait)
    // for this whole grid to finish before it reads anything.
    pdl_launch_dependents();
    // No CTA-wide barrier after this point: warps are independent workers.

    const int units_per_seq = p.Hkv * p.HB;
    const int w = blockIdx.x * p.warps + warp;
    if (w >= p.num_workers) return;
    if (p.zero_empty) {
        // no combine kernel follows: the workers write the zero rows of empty sequences
        for (int u = w; u < p.B * units_per_seq; u += p.num_workers) {
            const int b = u / units_per_seq;
            if (s_cum[b + 1] != s_cum[b]) continue;
            const int ulz = u - b * units_per_seq, kvh = ulz / p.HB, hb = ulz - (ulz / p.HB) * p.HB;
            write_zero_rows<D>(p, b, kvh * p.g + kMaxRows * hb, min(kMaxRows, p.g - kMaxRows * hb), lane);
        }
    }

    // This warp's run [ws, we) of sequence-tile positions, all for one unit-in-sequence ul
    // (kv head and head block).  Workers form groups of units_per_seq warps, one per (kv
    // head, head block); group grp owns an equal share of the positions of all sequences.
    // The warps of a group walk the same pages together, so the kv heads of a page are read
    // at about the same time.
    const int grp = w / units_per_seq;
    const int ul = w - grp * units_per_seq;
    const int ws = static_cast<int>(run_start(grp, s_cum[B], p.groups));
    const int we = static_cast<int>(run_start(grp + 1, s_cum[B], p.groups));
    if (ws >= we) return;

    const uint32_t bar0 = smem_u32(bars + warp * STAGES);
    const uint32_t wring = ring + static_cast<uint32_t>(warp) * STAGES * p.stage_bytes;  // unshared layout
    if constexpr (!SHARE) {
        if (lane == 0) {
#pragma unroll
            for (int s = 0; s < STAGES; ++s) mbar_init(bar0 + 8 * s, 1);
            fence_mbar_init();
        }
        __syncwarp();
    }

    const uint64_t pol_stream = l2_policy_evict_first();
    const uint64_t pol_keep = l2_policy_evict_last();

    const int kvh = ul / p.HB;
    const int hb = ul - kvh * p.HB;
    // Stage addresses.  Unshared: stage t of this warp is [K | V | Q] at wring + t * stage_bytes.
    // SHARE: the K/V ring of this warp's kv head (its leader is hb warps lower in the same
    // CTA: the host makes the warps per CTA a multiple of HB), and a Q ring of its own.
    const bool follower = SHARE && hb > 0;
    const uint32_t kv_step = SHARE ? 2 * G::kKVTileBytes : p.stage_bytes;
    const uint32_t q_step = SHARE ? ((p.q_box_bytes + 1023u) & ~1023u) : p.stage_bytes;
    const uint32_t kv_ring = SHARE ? ring + static_cast<uint32_t>(warp / p.HB) * STAGES * kv_step : wring;
    const uint32_t q_ring = SHARE ? ring + static_cast<uint32_t>(p.warps / p.HB) * STAGES * kv_step +
                                        static_cast<uint32_t>(warp) * STAGES * q_step
                                  : wring + 2 * G::kKVTileBytes;
    const uint32_t kv_bar0 = SHARE ? smem_u32(bars + (warp - hb) * STAGES) : bar0;
    const uint32_t empty0 = smem_u32(empties + (warp - hb) * STAGES);
    const int head0 = kvh * p.g + kMaxRows * hb;
    const int rows = min(kMaxRows, p.g - kMaxRows * hb);

    // LEAN: the lean per-tile form, which trims the instructions of a tile:
    // - the row sums of the bf16 weights come from an mma against a B of ones;
    // - 2^x is the SFU instruction;
    // - full tiles skip the masking selects;
    // - the rescale of the accumulators is skipped while no row's max grows;
    // - the page slot is a running cursor.
    // The plain form instead keeps:
    // - per-thread row sums, with the quad's partial sums added at the unit's end;
    // - exp2f;
    // - masking and rescale on every tile.
    // The host picks the form by measurement (B200, 268 MB of K/V, CUDA-graph replays):
    // - lean: D = 32, 64 and 128 (7-15% faster where per-tile latency binds);
    // - plain: D = 256, which sits at the 255-register cap (the lean form measured 2-3%
    //   slower there).  unit_kernel takes the plain form at D = 128 too (the lean form
    //   measured 1% slower on the llama8b shape with one CTA per unit).
    constexpr bool kLean = LEAN;

    // ---- producer state: next position to issue, its cursor, page-table window
    int pi = ws;
    int pb, pj, pn;
    decode_pos(ws, s_cum, B, pb, pj, pn);
    int pslot = (pj * kTile) % p.P;  // token slot of tile pj in its page (lean: stepped below)
    int wbase = ws;
    int32_t pg_cur = follower ? 0 : fetch_page(p, s_cum, ws + lane, we);
    int32_t pg_nxt = follower ? 0 : fetch_page(p, s_cum, ws + 32 + lane, we);

    bool stopped = false;  // the leader of a shared ring gave up on a release: no further issues
    auto issue_next = [&](int stage) {
        if (pi >= we || stopped) return;
        if (follower) {
            // this warp's Q rows only; an expect of 0 bytes keeps one phase per tile
            const bool qload = (pj == 0) || (pi == ws);
            if (lane == 0) {
                const uint32_t bar = bar0 + 8 * stage;
                const uint32_t qdst = q_ring + static_cast<uint32_t>(stage) * q_step;
                mbar_arrive_expect_tx(bar, qload ? p.q_box_bytes : 0u);
                if (qload) {
                    if constexpr (D == 32) tma_load_3d(qdst, &qmap, bar, 0, head0, pb, pol_keep);
                    else tma_load_4d(qdst, &qmap, bar, 0, head0, pb, 0, pol_keep);
                }
            }
            ++pi;
            if (pi < we) advance_pos(s_cum, pb, pj, pn);
            return;
        }
        if (SHARE && pi - ws >= STAGES) {
            // the followers have read the tile this stage held, STAGES tiles back.  If they
            // never release it (a follower gave up), issue nothing more: the stage may still
            // be read, and the consumer loop below stops at the first tile not issued.
            const int kk = pi - ws - STAGES;
            if (!warp_wait(empty0 + 8 * stage, static_cast<uint32_t>(kk / STAGES) & 1u, p.wait_ns, s_abort, p.flags)) {
                stopped = true;
                return;
            }
        }
        int off = pi - wbase;
        if (off >= 32) {
            pg_cur = pg_nxt;
            wbase += 32;
            off -= 32;
            pg_nxt = fetch_page(p, s_cum, wbase + 32 + lane, we);
        }
        const int32_t page = __shfl_sync(0xffffffffu, pg_cur, off);
        const int slot = kLean ? pslot : (pj * kTile) % p.P;
        const bool qload = (pj == 0) || (pi == ws);
        if (lane == 0) {
            if (page < 0 || page >= p.NP) atomicOr(p.flags, kFlagPageOOR);
            const uint32_t bar = bar0 + 8 * stage;
            const uint32_t sbase = kv_ring + static_cast<uint32_t>(stage) * kv_step;
            const uint32_t qdst = q_ring + static_cast<uint32_t>(stage) * q_step;
            mbar_arrive_expect_tx(bar, 2 * G::kKVTileBytes + (qload ? p.q_box_bytes : 0u));
            if constexpr (D == 32) {
                tma_load_4d(sbase, &kmap, bar, 0, kvh, slot, page, pol_stream);
                tma_load_4d(sbase + G::kKVTileBytes, &vmap, bar, 0, kvh, slot, page, pol_stream);
                if (qload) tma_load_3d(qdst, &qmap, bar, 0, head0, pb, pol_keep);
            } else {
                tma_load_5d(sbase, &kmap, bar, 0, kvh, slot, page, 0, pol_stream);
                tma_load_5d(sbase + G::kKVTileBytes, &vmap, bar, 0, kvh, slot, page, 0, pol_stream);
                if (qload) tma_load_4d(qdst, &qmap, bar, 0, head0, pb, 0, pol_keep);
            }
        }
        ++pi;
        if (pi < we) {
            advance_pos(s_cum, pb, pj, pn);
            if constexpr (kLean) pslot = (pj == 0 || pslot + kTile == p.P) ? 0 : pslot + kTile;
        }
    };

#pragma unroll
    for (int s = 0; s < STAGES; ++s) issue_next(s);

    // ---- consumer state
    int cb, cj, cn;
    decode_pos(ws, s_cum, B, cb, cj, cn);
    int seg_start = ws;
    int j_start = cj;
    TileAcc<D, LEAN> st;

    for (int i = ws; i < we; ++i) {
        const int k = i - ws;
        const int stage = k % STAGES;
        const uint32_t parity = static_cast<uint32_t>(k / STAGES) & 1u;
        const uint32_t sbase = kv_ring + static_cast<uint32_t>(stage) * kv_step;  // K, V
        const uint32_t qbase_t = q_ring + static_cast<uint32_t>(stage) * q_step;  // this warp's Q
        const bool unit_start = (cj == 0) || (i == ws);

        if (i >= pi || !warp_wait(kv_bar0 + 8 * stage, parity, p.wait_ns, s_abort, p.flags) ||
            (follower && !warp_wait(bar0 + 8 * stage, parity, p.wait_ns, s_abort, p.flags))) {
            // Gave up (this warp timed out, another warp of the CTA did, or this warp, as the
            // leader of a shared ring, stopped issuing): let this warp's own copies in flight
            // land, each wait bounded, then stop.
            *s_abort = 1u;
            for (int s = 0; s < STAGES; ++s) {
                const int t = i + s;
                if (t < pi) {
                    const int kk = t - ws;
                    warp_wait(bar0 + 8 * (kk % STAGES), static_cast<uint32_t>(kk / STAGES) & 1u, p.wait_ns / 8,
                              nullptr, nullptr);
                }
            }
            return;
        }

        if (unit_start) {
            seg_start = i;
            j_start = cj;
            st.reset();
            st.load_q(qbase_t, p.rows_max, rows, lane);
        }
        st.step(sbase, min(kTile, s_len[cb] - kTile * cj), p.scale_log2, lane);

        // ---- the stage is consumed: refill it with tile i + STAGES.  Each lane
        // orders its own shared-memory accesses (the tail zeroing included)
        // before the async-proxy write, then the warp syncs before lane 0 issues.
        fence_proxy_async_smem();
        __syncwarp();
        if (follower && lane == 0 && !p.test_skip_release) mbar_arrive(empty0 + 8 * stage);  // the leader may refill it
        issue_next(stage);

        // ---- end of this unit's run in this worker: write output or a partial
        const bool unit_end = (cj == cn - 1) || (i == we - 1);
        if (unit_end) {
            const bool direct = (j_start == 0) && (cj == cn - 1);
            if (direct) {
                st.write_out(p.out + cb * p.out_sb + head0 * p.out_sh, p.out_sh, rows, lane);
            } else {
                const int64_t slot = 2 * static_cast<int64_t>(w) + (seg_start == ws ? 0 : 1);
                st.write_part(p.o_part + slot * p.rows_max * D, D, p.ml_part + slot * p.rows_max * 2, rows, lane);
            }
        }
        if (i + 1 < we) advance_pos(s_cum, cb, cj, cn);
    }
}

// One CTA per unit (sequence b = unit / (Hkv * HB), kv head, head block), for launches in
// which every unit has an SM of its own (mode 2; the call is this one kernel), or, FIXED, one
// CTA per split of a unit with fixed splits (mode 1, k = ksplit: CTA u k + s takes split s,
// the tiles [s c, min((s + 1) c, n)) with c = ceil(n / min(k, n)), and writes the output when
// the unit has one non-empty split, else a partial for the combine kernel).  The two are
// separate instantiations: code for fixed splits in the mode-2 kernel measured 8% slower on
// the llama8b shape (47.3 against 43.9 us), with the mode-2 path itself unchanged.
//  * The mbarriers are set up before the wait on the previous grid.  After it, lane 0 of
//    each warp loads the sequence's length and claims its first STAGES + 1 tiles, loading
//    their page-table entries as the claims return.  (Deterministic first tiles, with all
//    those loads issued at once, measured 8% slower on the llama8b shape: the kv heads of
//    a sequence then read its pages in lockstep and whole sequences fell behind.)
//  * The warps claim the unit's 32-token tiles one at a time from a counter in shared
//    memory, each one tile ahead of its issue (the page-table entry of the claimed tile is
//    loaded while the tile before it streams), so a warp that streams faster takes more
//    tiles and the warps of the CTA end close together.
//  * Each warp keeps a running (max, sum, accumulator) over its tiles, writes it into its own
//    ring once its copies have landed, and the warps merge the parts through shared memory.
// Shared-memory layout: [full mbarriers, warps x STAGES][merge mbarrier][abort word, tile
// counter][claimed tile of each stage, warps x STAGES], then 1024-aligned rings of
// [K | V | Q] stages, one ring per warp.
template <int D, int STAGES, bool LEAN, bool FIXED>
__global__ void __launch_bounds__(32 * kMaxWarpsD<D, false>, 1)
    unit_kernel(const __grid_constant__ SplitParams p, const __grid_constant__ CUtensorMap kmap,
                const __grid_constant__ CUtensorMap vmap, const __grid_constant__ CUtensorMap qmap) {
    using G = Geometry<D>;
    extern __shared__ __align__(1024) uint8_t smem[];
    const int tid = threadIdx.x;
    const int lane = tid & 31;
    const int warp = tid >> 5;
    const int W = p.warps;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem);
    uint64_t* merge_bar = bars + W * STAGES;
    volatile uint32_t* s_abort = reinterpret_cast<volatile uint32_t*>(merge_bar + 1);
    uint32_t* s_next = reinterpret_cast<uint32_t*>(merge_bar + 1) + 1;
    int32_t* s_tile = reinterpret_cast<int32_t*>(merge_bar + 2);
    const uint32_t ring = (smem_u32(s_tile + W * STAGES) + 1023u) & ~1023u;
    const uint32_t wring = ring + static_cast<uint32_t>(warp) * STAGES * p.stage_bytes;
    const uint32_t bar0 = smem_u32(bars + warp * STAGES);
    int32_t* my_tile = s_tile + warp * STAGES;

    // ---- set-up that reads no global memory, overlapping the end of the previous kernel
    if (tid == 0) {
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
        prefetch_tensormap(&qmap);
        *s_abort = 0u;
        *s_next = 0u;
        mbar_init(smem_u32(merge_bar), 32u * static_cast<uint32_t>(W));  // every lane of every warp arrives
    }
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) mbar_init(bar0 + 8 * s, 1);
    }
    if (lane == 0) fence_mbar_init();
    __syncthreads();
    int nxt_t = 0;  // lane 0: the claimed tile that is issued next
    pdl_wait_prior_grid();
    pdl_launch_dependents();

    const int nsplit = FIXED ? p.ksplit : 1;
    const int u = FIXED ? blockIdx.x / nsplit : blockIdx.x;
    const int split = FIXED ? blockIdx.x - u * nsplit : 0;
    const int ups = p.Hkv * p.HB;
    const int b = u / ups;
    const int ul = u - b * ups;
    const int kvh = ul / p.HB;
    const int hb = ul - kvh * p.HB;
    const int head0 = kvh * p.g + kMaxRows * hb;
    const int rows = min(kMaxRows, p.g - kMaxRows * hb);
    // Contiguous KV (no page table): sequence b is "page" b of P = Lmax tokens, any length.
    const bool contig = p.page_table == nullptr;
    const int64_t cap = static_cast<int64_t>(p.MP) * p.P;  // tokens the page table can address
    const int32_t* pt_row = contig ? nullptr : p.page_table + static_cast<int64_t>(b) * p.pt_s0;
    const int tiles_per_page = contig ? 1 : p.P / kTile;
    const uint64_t pol_stream = l2_policy_evict_first();
    const uint64_t pol_keep = l2_policy_evict_last();

    // ---- producer state (lane 0): the next claimed tile and its page (a load in flight)
    auto page_of = [&](int t) -> int32_t {  // lane 0
        if (contig) return b;
        return (static_cast<int64_t>(t) * kTile < cap)
                   ? __ldcg(pt_row + static_cast<int64_t>(t / tiles_per_page) * p.pt_s1) : 0;
    };
    int32_t nxt_pg = 0;
    // Fixed splits take their tiles in a fixed order, so that a call's result does not depend
    // on timing: warp w streams the w-th contiguous share [w_lo, w_hi) of the split's tiles.
    int w_lo = 0, w_hi = 0;
    auto claim = [&]() {  // lane 0
        if constexpr (FIXED) {
            nxt_t = w_lo < w_hi ? w_lo++ : (1 << 30);
            nxt_pg = nxt_t < w_hi ? page_of(nxt_t) : 0;
        } else {
            nxt_t = static_cast<int>(atomicAdd(s_next, 1u));
            nxt_pg = page_of(nxt_t);
        }
    };
    // The split [t0, t1) of n tiles (fixed splits), and how many splits are not empty.
    auto split_range = [&](int n, int& t0, int& t1, int& nk) {
        if (!FIXED || n == 0) {
            t0 = 0;
            t1 = n;
            nk = 1;
            return;
        }
        const int S = max(1, min(nsplit, n));
        const int c = (n + S - 1) / S;
        t0 = min(split * c, n);
        t1 = min(t0 + c, n);
        nk = (n + c - 1) / c;
    };
    // lane 0: the sequence's length, then this warp's first STAGES + 1 claims with their pages
    int L = 0;
    int t0[STAGES];
    int32_t pg0[STAGES];
    if (lane == 0) {
        L = __ldcg(p.seq_lens + b);
        auto clamp_len = [&]() {
            uint32_t len_flags = 0;
            if (L < 0) {
                L = 0;
                len_flags |= kFlagLenNegative;
            }
            if (L > cap) {
                L = static_cast<int>(cap);
                len_flags |= kFlagLenClamped;
            }
            if (len_flags && warp == 0 && split == 0) atomicOr(p.flags, len_flags);
        };
        if constexpr (FIXED) {
            // fixed splits: the split's tiles depend on the length, so it comes first
            clamp_len();
            int s0, s1, nk_;
            split_range((L + kTile - 1) / kTile, s0, s1, nk_);
            const int cnt = s1 - s0, c = (cnt + W - 1) / W;
            w_lo = s0 + min(cnt, warp * c);
            w_hi = s0 + min(cnt, (warp + 1) * c);
        }
#pragma unroll
        for (int s = 0; s < STAGES; ++s) {
            claim();
            t0[s] = nxt_t;
            pg0[s] = nxt_pg;
        }
        claim();
        if constexpr (!FIXED) clamp_len();
    }
    L = __shfl_sync(0xffffffffu, L, 0);
    const int n = (L + kTile - 1) / kTile;
    int t_lo, t_hi, nk;  // this CTA's tiles [t_lo, t_hi) and the unit's non-empty splits
    split_range(n, t_lo, t_hi, nk);
    // an empty split writes nothing (the unit's output, zeros for an empty sequence, comes
    // from split 0)
    if (FIXED && t_lo >= t_hi && split > 0) return;

    // Issue tile t (page pg) into stage `stage`, with the Q rows on this warp's first tile.
    auto issue = [&](int stage, int t, int32_t pg, bool qload) {  // lane 0
        if (pg < 0 || pg >= p.NP) atomicOr(p.flags, kFlagPageOOR);
        my_tile[stage] = t;
        const uint32_t bar = bar0 + 8 * stage;
        const uint32_t sbase = wring + static_cast<uint32_t>(stage) * p.stage_bytes;
        const int slot = contig ? t * kTile : (t % tiles_per_page) * kTile;
        mbar_arrive_expect_tx(bar, 2 * G::kKVTileBytes + (qload ? p.q_box_bytes : 0u));
        if constexpr (D == 32) {
            tma_load_4d(sbase, &kmap, bar, 0, kvh, slot, pg, pol_stream);
            tma_load_4d(sbase + G::kKVTileBytes, &vmap, bar, 0, kvh, slot, pg, pol_stream);
            if (qload) tma_load_3d(sbase + 2 * G::kKVTileBytes, &qmap, bar, 0, head0, b, pol_keep);
        } else {
            tma_load_5d(sbase, &kmap, bar, 0, kvh, slot, pg, 0, pol_stream);
            tma_load_5d(sbase + G::kKVTileBytes, &vmap, bar, 0, kvh, slot, pg, 0, pol_stream);
            if (qload) tma_load_4d(sbase + 2 * G::kKVTileBytes, &qmap, bar, 0, head0, b, 0, pol_keep);
        }
    };
    int issued = 0;  // stages issued so far (warp-uniform)
    if (lane == 0) {
#pragma unroll
        for (int s = 0; s < STAGES; ++s) {
            if (t0[s] < t_hi) {
                issue(s, t0[s], pg0[s], s == 0);
                ++issued;
            }
        }
    }
    issued = __shfl_sync(0xffffffffu, issued, 0);

    TileAcc<D, LEAN> st;
    st.reset();
    for (int k = 0; k < issued; ++k) {
        const int stage = k % STAGES;
        const uint32_t sbase = wring + static_cast<uint32_t>(stage) * p.stage_bytes;
        if (!warp_wait(bar0 + 8 * stage, static_cast<uint32_t>(k / STAGES) & 1u, p.wait_ns, s_abort, p.flags)) {
            // gave up: let this warp's other copies in flight land (bounded), then stop
            *s_abort = 1u;
            for (int kk = k + 1; kk < issued; ++kk)
                warp_wait(bar0 + 8 * (kk % STAGES), static_cast<uint32_t>(kk / STAGES) & 1u, p.wait_ns / 8, nullptr,
                          nullptr);
            return;
        }
        const int t = my_tile[stage];
        if (k == 0) st.load_q(sbase + 2 * G::kKVTileBytes, p.rows_max, rows, lane);
        st.step(sbase, min(kTile, L - kTile * t), p.scale_log2, lane);
        // the stage is consumed: refill it with the claimed tile, if any, and claim the next
        fence_proxy_async_smem();
        __syncwarp();
        int more = 0;
        if (lane == 0 && nxt_t < t_hi) {
            issue(stage, nxt_t, nxt_pg, false);
            claim();
            more = 1;
        }
        issued += __shfl_sync(0xffffffffu, more, 0);
    }

    // ---- this warp's part (empty when it got no tile) into its own ring, then the merge
    float* const own = reinterpret_cast<float*>(smem + (wring - smem_u32(smem)));
    st.write_part(own + 2 * kMaxRows, kPartStride<D>, own, rows, lane);
    mbar_arrive(smem_u32(merge_bar));
    if (!warp_wait(smem_u32(merge_bar), 0u, p.wait_ns, s_abort, p.flags)) return;
    // one non-empty split: the output; else this split's partial
    const int64_t slot = (FIXED && nk > 1) ? static_cast<int64_t>(u) * nsplit + split : -1;
    unit_merge<D>(p, smem + (ring - smem_u32(smem)), static_cast<uint32_t>(STAGES) * p.stage_bytes, b, head0, rows,
                  warp, W, lane, slot);
}

constexpr int kCombineBatch = 4;  // partial slots whose loads a warp issues together

// One CTA per (unit, head row).  Merges the row's partials:
//   M = max_s m_s over non-empty partials,
//   out = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s.
// The CTA's warps split the unit's partial slots and each keeps a running
// (max, sum, acc) over its share, loading kCombineBatch slots at a time; each
// lane owns float4 columns of the row.  The warps' states are merged through
// shared memory.  In balanced mode it also writes zeros for empty sequences.  W warps
// (4, 8 or 16, from the partials a unit is expected to have: one batch per warp).
template <int D, int W>
__global__ void __launch_bounds__(32 * W) combine_kernel(const __grid_constant__ CombineParams p) {
    constexpr int kCombineWarps = W;
    constexpr int kCols = D / 4;                 // float4 columns of a row
    constexpr int kPerLane = (kCols + 31) / 32;  // float4 columns per lane
    __shared__ float4 s_acc[kCombineWarps][kCols];
    __shared__ float s_m[kCombineWarps], s_den[kCombineWarps];

    // Every CTA of this grid is resident once it gets here, so the next kernel in
    // the stream may begin launching (it waits for this grid before reading).
    pdl_launch_dependents();

    const int u = blockIdx.x;
    const int r = blockIdx.y;
    const int units_per_seq = p.Hkv * p.HB;
    const int b = u / units_per_seq;
    const int ul = u - b * units_per_seq;
    const int kvh = ul / p.HB;
    const int hb = ul - kvh * p.HB;
    const int rows = min(kMaxRows, p.g - kMaxRows * hb);
    if (r >= rows) return;
    const int head = kvh * p.g + kMaxRows * hb + r;
    __nv_bfloat16* orow = p.out + b * p.out_sb + head * p.out_sh;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // Tile counts of the sequences, clamped as the split kernel clamps them, and their
    // prefix sums at b and over all B.  This runs before the wait on the split grid:
    // seq_lens is not written by it, and this grid cannot start before every split CTA
    // has passed its own wait on the kernel before it, so seq_lens is final here.  It
    // takes one dependent load off the path that follows the split grid's end.
    __shared__ int s_pre[kCombineWarps], s_tot[kCombineWarps], s_nb;
    {
        const int64_t cap = static_cast<int64_t>(p.MP) * p.P;
        int pre = 0, tot = 0;
        for (int i = tid; i < p.B; i += blockDim.x) {
            int L = __ldcg(p.seq_lens + i);
            L = L < 0 ? 0 : (L > cap ? static_cast<int>(cap) : L);
            const int t = (L + kTile - 1) / kTile;
            tot += t;
            if (i < b) pre += t;
            if (i == b) s_nb = t;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            pre += __shfl_xor_sync(0xffffffffu, pre, o);
            tot += __shfl_xor_sync(0xffffffffu, tot, o);
        }
        if (lane == 0) {
            s_pre[warp] = pre;
            s_tot[warp] = tot;
        }
        __syncthreads();
    }
    int cum_b = 0, cum_B = 0;
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) {
        cum_b += s_pre[w];
        cum_B += s_tot[w];
    }
    const int n = s_nb;

    pdl_wait_prior_grid();
    if (n == 0) {
        if (p.mode == 0)
            for (int c = tid; c < kCols; c += blockDim.x) *reinterpret_cast<uint2*>(orow + 4 * c) = make_uint2(0u, 0u);
        return;
    }

    // The unit's partial slots, numbered k = 0 .. nk-1.  Balanced mode: the groups
    // whose shares of the sequence-tile positions meet sequence b; group g's warp
    // for this unit is g * units_per_seq + ul.
    int nk, g_first = 0, first_slot_fixed = 0;
    int64_t total = 0, Sb = 0;
    if (p.mode == 0) {
        total = cum_B;
        Sb = cum_b;
        g_first = worker_of(Sb, total, p.groups);
        const int g_last = worker_of(Sb + n - 1, total, p.groups);
        if (g_first == g_last) return;  // one warp covered it and wrote the output
        nk = g_last - g_first + 1;
    } else {
        const int S = min(p.ksplit, n);
        const int c = (n + S - 1) / S;
        nk = (n + c - 1) / c;
        if (nk == 1) return;
        first_slot_fixed = u * p.ksplit;
    }
    // slot of partial k, or -1 for a group whose share is empty (it wrote nothing)
    auto slot_of = [&](int k) -> int64_t {
        if (p.mode != 0) return first_slot_fixed + k;
        const int g = g_first + k;
        const int64_t a = run_start(g, total, p.groups);
        if (a == run_start(g + 1, total, p.groups)) return -1;
        const int64_t w = static_cast<int64_t>(g) * units_per_seq + ul;
        return 2 * w + ((k == 0 && a != Sb) ? 1 : 0);
    };

    float M = -INFINITY, den = 0.f;
    float4 acc[kPerLane];
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int k0 = warp; k0 < nk; k0 += kCombineBatch * kCombineWarps) {
        float2 ml[kCombineBatch];
        float4 o[kCombineBatch][kPerLane];
#pragma unroll
        for (int t = 0; t < kCombineBatch; ++t) {
            const int k = k0 + t * kCombineWarps;
            const int64_t slot = k < nk ? slot_of(k) : -1;
            ml[t] = make_float2(-INFINITY, 0.f);
            if (slot >= 0) {
                ml[t] = *reinterpret_cast<const float2*>(p.ml_part + (slot * p.rows_max + r) * 2);
                const float4* src = reinterpret_cast<const float4*>(p.o_part + (slot * p.rows_max + r) * D);
#pragma unroll
                for (int j = 0; j < kPerLane; ++j) {
                    const int c = lane + 32 * j;
                    o[t][j] = c < kCols ? src[c] : make_float4(0.f, 0.f, 0.f, 0.f);
                }
            }
        }
#pragma unroll
        for (int t = 0; t < kCombineBatch; ++t) {
            if (!(ml[t].y > 0.f)) continue;  // empty split or no slot
            if (ml[t].x > M) {
                const float sc = exp2f(M - ml[t].x);  // 0 while M is -inf (acc and den are 0 then)
                den *= sc;
#pragma unroll
                for (int j = 0; j < kPerLane; ++j) {
                    acc[j].x *= sc;
                    acc[j].y *= sc;
                    acc[j].z *= sc;
                    acc[j].w *= sc;
                }
                M = ml[t].x;
            }
            const float wgt = exp2f(ml[t].x - M);
            den += wgt * ml[t].y;
#pragma unroll
            for (int j = 0; j < kPerLane; ++j) {
                acc[j].x += wgt * o[t][j].x;
                acc[j].y += wgt * o[t][j].y;
                acc[j].z += wgt * o[t][j].z;
                acc[j].w += wgt * o[t][j].w;
            }
        }
    }
#pragma unroll
    for (int j = 0; j < kPerLane; ++j) {
        const int c = lane + 32 * j;
        if (c < kCols) s_acc[warp][c] = acc[j];
    }
    if (lane == 0) {
        s_m[warp] = M;
        s_den[warp] = den;
    }
    __syncthreads();

    float Mt = -INFINITY;
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w)
        if (s_den[w] > 0.f) Mt = fmaxf(Mt, s_m[w]);
    float wt[kCombineWarps];
    float dsum = 0.f;
#pragma unroll
    for (int w = 0; w < kCombineWarps; ++w) {
        wt[w] = s_den[w] > 0.f ? exp2f(s_m[w] - Mt) : 0.f;
        dsum += wt[w] * s_den[w];
    }
    const float inv = 1.f / dsum;
    for (int c = tid; c < kCols; c += blockDim.x) {
        float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w = 0; w < kCombineWarps; ++w) {
            if (wt[w] == 0.f) continue;
            const float4 a = s_acc[w][c];
            t.x += wt[w] * a.x;
            t.y += wt[w] * a.y;
            t.z += wt[w] * a.z;
            t.w += wt[w] * a.w;
        }
        uint2 packed;
        packed.x = pack_bf16x2(t.x * inv, t.y * inv);
        packed.y = pack_bf16x2(t.z * inv, t.w * inv);
        *reinterpret_cast<uint2*>(orow + 4 * c) = packed;
    }
}

// The unit's partial slots in the combine: which slots hold its parts, as the split kernel
// wrote them (balanced groups, or fixed splits), and the unit's sequence facts.
struct UnitSlots {
    int n = 0;         // tiles of the unit's sequence (0: empty sequence)
    int nk = 0;        // partial slots, numbered k = 0 .. nk-1 (<= 1: nothing to merge)
    int g_first = 0;   // balanced: the first group meeting the sequence
    int64_t total = 0, Sb = 0;
    int64_t first_fixed = 0;
};

// Balanced mode: the groups whose shares of the sequence-tile positions meet sequence b
// (cum_b = tiles before b, cum_B = all tiles); fixed mode: the unit's non-empty splits.
__device__ __forceinline__ UnitSlots unit_slots(const CombineParams& p, int u, int n, int cum_b, int cum_B) {
    UnitSlots s;
    s.n = n;
    if (n == 0) return s;
    if (p.mode == 0) {
        s.total = cum_B;
        s.Sb = cum_b;
        s.g_first = worker_of(s.Sb, s.total, p.groups);
        const int g_last = worker_of(s.Sb + n - 1, s.total, p.groups);
        s.nk = g_last - s.g_first + 1;  // 1: one warp covered it and wrote the output
    } else {
        const int S = min(p.ksplit, n);
        const int c = (n + S - 1) / S;
        s.nk = (n + c - 1) / c;
        s.first_fixed = static_cast<int64_t>(u) * p.ksplit;
    }
    return s;
}

// Slot of partial k of unit-in-sequence ul, or -1 for a group whose share is empty.
__device__ __forceinline__ int64_t slot_of(const CombineParams& p, const UnitSlots& s, int ul, int k) {
    if (p.mode != 0) return s.first_fixed + k;
    const int g = s.g_first + k;
    const int64_t a = run_start(g, s.total, p.groups);
    if (a == run_start(g + 1, s.total, p.groups)) return -1;
    const int64_t w = static_cast<int64_t>(g) * p.Hkv * p.HB + ul;
    return 2 * w + ((k == 0 && a != s.Sb) ? 1 : 0);
}

// Combine for plans with few partials per unit (large batches): a grid of at most a few
// CTAs per SM, each taking units u = blockIdx.x, + gridDim.x, ...  Every CTA first turns
// seq_lens into the tiles' prefix sums in shared memory (before the wait on the split grid:
// seq_lens is not written by it), so a unit that one warp covered, or an empty one, costs no
// global access after the wait.  A unit to merge has each warp merge whole rows on its own
// (all of a row's partial slots, kCombineBatch loads in flight).  Same merge as
// combine_kernel.  Dynamic shared memory: (B + 1) int32.
template <int D, int W>
__global__ void __launch_bounds__(32 * W) combine_unit_kernel(const __grid_constant__ CombineParams p) {
    constexpr int kCols = D / 4;                 // float4 columns of a row
    constexpr int kPerLane = (kCols + 31) / 32;  // float4 columns per lane
    extern __shared__ int32_t s_cum[];           // [B + 1]: tiles of the sequences before b
    __shared__ int s_wsum[W];
    pdl_launch_dependents();
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int B = p.B;
    {
        // each thread takes `per` consecutive sequences; block-wide exclusive scan
        const int64_t cap = static_cast<int64_t>(p.MP) * p.P;
        const int per = (B + 32 * W - 1) / (32 * W);
        const int lo = tid * per, hi = min(lo + per, B);
        int sum = 0;
        for (int i = lo; i < hi; ++i) {
            int L = __ldcg(p.seq_lens + i);
            L = L < 0 ? 0 : (L > cap ? static_cast<int>(cap) : L);
            const int t = (L + kTile - 1) / kTile;
            s_cum[i + 1] = t;
            sum += t;
        }
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += v;
        }
        if (lane == 31) s_wsum[warp] = incl;
        __syncthreads();
        int run = incl - sum;
        for (int w = 0; w < warp; ++w) run += s_wsum[w];
        for (int i = lo; i < hi; ++i) {
            run += s_cum[i + 1];
            s_cum[i + 1] = run;
        }
        if (tid == 0) s_cum[0] = 0;
        __syncthreads();
    }
    pdl_wait_prior_grid();
    const int ups = p.Hkv * p.HB;
    const int units = B * ups;
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int b = u / ups;
        const int ul = u - b * ups;
        const int kvh = ul / p.HB;
        const int hb = ul - kvh * p.HB;
        const int rows = min(kMaxRows, p.g - kMaxRows * hb);
        const int head0 = kvh * p.g + kMaxRows * hb;
        const UnitSlots us = unit_slots(p, u, s_cum[b + 1] - s_cum[b], s_cum[b], s_cum[B]);
        if (us.n == 0) {
            if (p.mode == 0)  // balanced mode: the combine writes the rows of empty sequences
                for (int i = tid; i < rows * kCols; i += blockDim.x) {
                    const int r = i / kCols, c = i - r * kCols;
                    *reinterpret_cast<uint2*>(p.out + b * p.out_sb + (head0 + r) * p.out_sh + 4 * c) =
                        make_uint2(0u, 0u);
                }
            continue;
        }
        if (us.nk <= 1) continue;

        for (int r = warp; r < rows; r += W) {
            float M = -INFINITY, den = 0.f;
            float4 acc[kPerLane];
#pragma unroll
            for (int j = 0; j < kPerLane; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int k0 = 0; k0 < us.nk; k0 += kCombineBatch) {
                float2 ml[kCombineBatch];
                float4 o[kCombineBatch][kPerLane];
#pragma unroll
                for (int t = 0; t < kCombineBatch; ++t) {
                    const int kk = k0 + t;
                    const int64_t slot = kk < us.nk ? slot_of(p, us, ul, kk) : -1;
                    ml[t] = make_float2(-INFINITY, 0.f);
                    if (slot >= 0) {
                        ml[t] = *reinterpret_cast<const float2*>(p.ml_part + (slot * p.rows_max + r) * 2);
                        const float4* src = reinterpret_cast<const float4*>(p.o_part + (slot * p.rows_max + r) * D);
#pragma unroll
                        for (int j = 0; j < kPerLane; ++j) {
                            const int c = lane + 32 * j;
                            o[t][j] = c < kCols ? src[c] : make_float4(0.f, 0.f, 0.f, 0.f);
                        }
                    }
                }
#pragma unroll
                for (int t = 0; t < kCombineBatch; ++t) {
                    if (!(ml[t].y > 0.f)) continue;  // empty split or no slot
                    if (ml[t].x > M) {
                        const float sc = exp2f(M - ml[t].x);  // 0 while M is -inf (acc and den are 0 then)
                        den *= sc;
#pragma unroll
                        for (int j = 0; j < kPerLane; ++j) {
                            acc[j].x *= sc;
                            acc[j].y *= sc;
                            acc[j].z *= sc;
                            acc[j].w *= sc;
                        }
                        M = ml[t].x;
                    }
                    const float wgt = exp2f(ml[t].x - M);
                    den += wgt * ml[t].y;
#pragma unroll
                    for (int j = 0; j < kPerLane; ++j) {
                        acc[j].x += wgt * o[t][j].x;
                        acc[j].y += wgt * o[t][j].y;
                        acc[j].z += wgt * o[t][j].z;
                        acc[j].w += wgt * o[t][j].w;
                    }
                }
            }
            const float inv = den > 0.f ? 1.f / den : 0.f;
            __nv_bfloat16* orow = p.out + b * p.out_sb + (head0 + r) * p.out_sh;
#pragma unroll
            for (int j = 0; j < kPerLane; ++j) {
                const int c = lane + 32 * j;
                if (c < kCols) {
                    uint2 packed;
                    packed.x = pack_bf16x2(acc[j].x * inv, acc[j].y * inv);
                    packed.y = pack_bf16x2(acc[j].z * inv, acc[j].w * inv);
                    *reinterpret_cast<uint2*>(orow + 4 * c) = packed;
                }
            }
        }
    }
}

}  // namespace apd
