// apd_prefill_tc.cuh -- multi-query (chunked prefill) attention over the paged
// bf16 KV cache on the sm_100a fifth-generation tensor cores (tcgen05 + TMEM).
//
// Same operation as apd_prefill.cuh (AstrAI commit log of
// csrc/kernels/attn_paged_decode.cu: prefill over the paged KV policy with the
// unified causal_offset and 2-D / 3-D masks); this is the dense-contraction
// design for B200.  Two kernels:
//
//  * prefill_tc2_kernel -- two 128-row Q tiles per CTA (used when a kv head has
//    more than 128 query rows, D = 32, 64, 128); described with its code below.
//  * prefill_tc_kernel -- one 128-row Q tile per CTA (D = 256, and fewer rows):
//
//  - A CTA owns M = 128 query rows of one (sequence b, kv head), the
//    (query i, head-in-group hh) pairs in query-major order (row = i * g + hh),
//    so the g heads of the kv head share every K/V tile.
//  - Warp 8 (producer) resolves the pages of each tile of N keys and issues the
//    TMA loads of the K and V tiles, 32 tokens per box, into two STAGES-deep
//    rings laid out as the swizzled canonical operand layouts of the tensor core
//    (OperandGeom: [D/64][N][64] blocks with the 128-byte swizzle, or for
//    D = 32 one block of 64-byte rows with the 64-byte swizzle).
//  - Warp 9 lane 0 (MMA issuer) runs S_j = Q K_j^T (M=128, N keys, K=D; both
//    operands K-major) into one of two TMEM S buffers and O += P_j V_j
//    (M=128, N=D, K=N keys; V is the MN-major B operand) into a TMEM O
//    accumulator; tcgen05.commit arrives on the mbarriers that free the K/V
//    stages and hand S and O to the softmax warps.  The next tile's Q K^T runs
//    while the softmax warps work on the current one.
//  - Warps 0-7 (softmax): TMEM lane r is query row r; warps w and w + 4 both
//    read lane quadrant w (a warp may only reach the quadrant of its warp index
//    mod 4) and each takes half of the row's columns, so every SM sub-partition
//    runs two softmax warps.  A thread owns one row half: row maximum and sum
//    need no shuffles, only one exchange of the two halves' maxima per tile
//    through shared memory and an mbarrier.  The warps load S from TMEM, apply
//    the visibility (length, causal offset, mask), keep a lazily updated running
//    maximum (O in TMEM is rescaled only when a row's maximum grows by more than
//    2^8), write P = 2^(s * scale * log2 e - max) (MUFU ex2, the scale folded
//    into one FFMA) as bf16 into shared memory in the swizzled A layout, and in
//    the epilogue read O from TMEM, divide by the row sum and store bf16.
//
// In both, every mbarrier wait is bounded; a wait that runs out raises a shared
// abort flag that every role polls, the producer and the MMA issuer then wait
// (bounded) for their own copies and MMAs in flight, and all warps meet before
// the TMEM columns are freed.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "apd_kernels.cuh"
#include "apd_prefill.cuh"
#include "apd_ptx.cuh"

namespace apd {

// ------------------------------------------------------------------ tcgen05
__device__ __forceinline__ void tc_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem), "r"(ncols)
                 : "memory");
}
__device__ __forceinline__ void tc_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tc_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// Arrive once on `bar` when every tcgen05 operation this thread issued so far has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
                 : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, bf16 in, fp32 accumulate.
__device__ __forceinline__ void tc_mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void tc_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tc_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tc_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 TMEM lanes x 32 columns of 32 bits: thread t of the warp gets lane (lane of
// taddr) + t, columns [column of taddr, +32).
__device__ __forceinline__ void tc_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
}
__device__ __forceinline__ void tc_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
        "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
        "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
        "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}

// Shared-memory matrix descriptor of a 128-byte-swizzled operand tile (sm_100
// layout: start address >> 4 in bits 0-13, leading byte offset >> 4 in 16-29,
// stride byte offset >> 4 in 32-45, descriptor version 1 in 46-47, base offset 0,
// swizzle mode 2 = 128 B in 61-63).  The tile's 1024-byte swizzle atoms must be
// 1024-byte aligned; a start address inside an atom (a K step of 32 bytes) is
// allowed because the swizzle is applied to the computed address bits.
//   K-major : 8-row groups at `sbo` bytes; `lbo` unused (1).
//   MN-major: 64-element column blocks at `lbo` bytes, 8-row groups of K at `sbo`.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// The same for the 64-byte swizzle (mode 4), whose atoms are 8 rows of 64 bytes: the
// layout of operands with 32-element rows (head dim 32).
__device__ __forceinline__ uint64_t sw64_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16) |
           (static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (4ull << 61);
}

// Staging geometry of a [rows][D] bf16 operand: column blocks of kCols elements
// (64 with the 128-byte swizzle; the whole row, 32, with the 64-byte swizzle for
// D = 32), each block [rows][kCols] with kRowBytes-byte rows.
template <int D>
struct OperandGeom {
    static constexpr int kCols = D >= 64 ? 64 : D;
    static constexpr int kRowBytes = 2 * kCols;
    static constexpr int kBlk = D / kCols;
    static constexpr int kChunks = kRowBytes / 16;  // 16-byte chunks per row of a block
    static constexpr uint32_t kSbo = 8 * kRowBytes;  // 8-row groups
    static_assert(D == 32 || D % 64 == 0, "head dim");
    // physical 16-byte chunk of logical chunk c in row `row` of a block
    __device__ static constexpr int swz(int row, int c) { return D >= 64 ? (c ^ (row & 7)) : (c ^ ((row >> 1) & 3)); }
    __device__ static uint64_t desc(uint32_t saddr, uint32_t lbo) {
        if constexpr (D >= 64) return sw128_desc(saddr, lbo, kSbo);
        else return sw64_desc(saddr, lbo, kSbo);
    }
    // K-major operand [rows][D] staged as kBlk blocks of [rows][kCols]: start of the 16-
    // element K step ks
    __device__ static constexpr uint32_t kstep(int ks, int rows) {
        return static_cast<uint32_t>((ks / (kCols / 16)) * rows * kRowBytes + (ks % (kCols / 16)) * 32);
    }
};

// Instruction descriptor of tcgen05.mma kind::f16 with bf16 A and B, fp32 D,
// A K-major, B K-major or MN-major, shape M x N (N % 16 == 0 for M = 128).
constexpr uint32_t bf16_idesc(int M, int N, bool b_mn_major) {
    return (1u << 4)                               // D format: fp32
           | (1u << 7)                             // A format: bf16
           | (1u << 10)                            // B format: bf16
           | ((b_mn_major ? 1u : 0u) << 16)        // B major-ness
           | (static_cast<uint32_t>(N >> 3) << 17)  // N / 8
           | (static_cast<uint32_t>(M >> 4) << 24); // M / 16
}

// ---- packed fp32 pairs (sm_100a f32x2 arithmetic) and a 3-input maximum
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
    uint64_t r;
    asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
    return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
    asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
    uint64_t d;
    asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
    return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
    uint64_t d;
    asm("add.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
    return d;
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Parts in which a softmax warpgroup of the two-tile kernel hands P over to the MMA
// issuer (the first parts' P V runs while the later parts' exponentials are computed).
// Chunk workload (D = 128): 1 part 185.2 us, 2 parts 183.6 us, 4 parts 181.7 us.
#ifndef APD_PREFILL_P_PARTS
#define APD_PREFILL_P_PARTS 4
#endif

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d)
                 : "memory");
}

// ---- pieces shared by the tensor-core prefill kernels

// Q rows [row_first, row_first + 128) of (sequence b, kv head kvh), the (query, head-in-
// group) pairs row = i * g + hh, into the 128-byte-swizzled K-major A layout
// [D/64][128][64] at q_s; rows >= R are zeros.  Threads tid (of nthreads) share the copy.
template <int D>
__device__ __forceinline__ void stage_q_tile(uint32_t q_s, const PrefillParams& p, int b, int kvh, int row_first,
                                             int R, int tid, int nthreads) {
    using O = OperandGeom<D>;
    constexpr int M = 128;
    // Loads issued together before their stores: one round trip per batch rather than per
    // 16-byte chunk (the shared store's memory clobber keeps the compiler from hoisting the
    // next load).  Chunk workload, D = 128: 180.4 -> 170.8 us with 8; 16 measured 179 us.
    constexpr int kBatch = 8;
    for (int idx0 = tid; idx0 < M * (D / 8); idx0 += kBatch * nthreads) {
        uint4 v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int idx = idx0 + u * nthreads;
            const int row = idx / (D / 8), ch = idx % (D / 8);
            const int rq = row_first + row;
            v[u] = make_uint4(0u, 0u, 0u, 0u);
            if (idx < M * (D / 8) && rq < R) {
                const int i = rq / p.g, hh = rq - i * p.g;
                v[u] = __ldg(reinterpret_cast<const uint4*>(p.q + b * p.q_sb + i * p.q_si + (kvh * p.g + hh) * p.q_sh +
                                                            ch * 8));
            }
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
            const int idx = idx0 + u * nthreads;
            if (idx >= M * (D / 8)) break;
            const int row = idx / (D / 8), ch = idx % (D / 8);
            st_shared_v4(q_s + static_cast<uint32_t>((ch / O::kChunks) * (M * O::kRowBytes) + row * O::kRowBytes +
                                                     (O::swz(row, ch % O::kChunks) << 4)),
                         v[u].x, v[u].y, v[u].z, v[u].w);
        }
    }
}

// Zeroes rows [v0, N) of a V tile staged as OperandGeom blocks (the swizzle only permutes
// 16-byte chunks within a row, so whole rows are cleared in place).
template <int D, int N>
__device__ __forceinline__ void zero_v_rows(uint32_t vb, int v0, int tid, int nthreads) {
    using O = OperandGeom<D>;
    constexpr int kPerRow = O::kBlk * O::kChunks;
    for (int idx = tid; idx < (N - v0) * kPerRow; idx += nthreads) {
        const int row = v0 + idx / kPerRow, rest = idx % kPerRow;
        st_shared_zero16(vb + static_cast<uint32_t>((rest / O::kChunks) * (N * O::kRowBytes) + row * O::kRowBytes +
                                                    ((rest % O::kChunks) << 4)));
    }
}

// Epilogue of one row: NC columns of O from TMEM at taddr (this thread's lane), times inv,
// as bf16 to orow.  The TMEM loads are warp-collective, so every lane loads; only rows
// that exist store.  With no tile processed (have_o false) the row is zeros.
template <int NC>
__device__ __forceinline__ void store_o_row(uint32_t taddr, bool have_o, float inv, bool row_ok,
                                            __nv_bfloat16* orow) {
#pragma unroll 1
    for (int c = 0; c < NC / 32; ++c) {
        uint32_t o[32];
        if (have_o) {
            tc_ld32(taddr + static_cast<uint32_t>(32 * c), o);
            tc_wait_ld();
        } else {
#pragma unroll
            for (int e = 0; e < 32; ++e) o[e] = 0u;
        }
        if (row_ok) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                uint4 w;
                w.x = pack_bf16x2(__uint_as_float(o[8 * e + 0]) * inv, __uint_as_float(o[8 * e + 1]) * inv);
                w.y = pack_bf16x2(__uint_as_float(o[8 * e + 2]) * inv, __uint_as_float(o[8 * e + 3]) * inv);
                w.z = pack_bf16x2(__uint_as_float(o[8 * e + 4]) * inv, __uint_as_float(o[8 * e + 5]) * inv);
                w.w = pack_bf16x2(__uint_as_float(o[8 * e + 6]) * inv, __uint_as_float(o[8 * e + 7]) * inv);
                *reinterpret_cast<uint4*>(orow + 32 * c + 8 * e) = w;
            }
        }
    }
}

// Tile shape and shared-memory / TMEM layout per head dim.
template <int D>
struct TcShape {
    static constexpr int kM = 128;                    // query rows per CTA (TMEM lanes)
    static constexpr int kN = (D == 256) ? 64 : 128;  // keys per tile
    static constexpr int kStages = (D == 32) ? 6 : (D == 64) ? 4 : 2;
    static constexpr int kSoftmaxWarps = 8;  // two per TMEM lane quadrant, half a row's columns each
    static constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
    static constexpr int kProducerWarp = kSoftmaxWarps, kMmaWarp = kSoftmaxWarps + 1;
    static constexpr int kThreads = 32 * (kSoftmaxWarps + 2);
    static constexpr uint32_t kQBytes = kM * D * 2;
    static constexpr uint32_t kKVBytes = kN * D * 2;  // one K (or V) tile
    static constexpr uint32_t kPBytes = kM * kN * 2;
    static constexpr uint32_t kQOff = 0;
    static constexpr uint32_t kKOff = kQBytes;
    static constexpr uint32_t kVOff = kKOff + kStages * kKVBytes;
    static constexpr uint32_t kPOff = kVOff + kStages * kKVBytes;
    static constexpr uint32_t kTileBytes = kPOff + kPBytes;
    // 4 KB header (barriers, TMEM address, abort flag, the row-maximum and row-sum
    // exchange between the two warps of a row), up to 1 KB to reach 1024-byte
    // alignment, then the tiles
    static constexpr uint32_t kHeaderBytes = 4096;
    static constexpr uint32_t kSmemBytes = kHeaderBytes + 1024 + kTileBytes;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0;       // two S buffers: columns [0, 2N)
    static constexpr uint32_t kColO = 2 * kN;  // O: columns [2N, 2N + D)
    static_assert(2 * kN + D <= 512, "TMEM columns");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kSmemBytes > 232448 / 2, "one CTA per SM, so the 512 TMEM columns are always free");
};

// Bounded mbarrier wait that also gives up when another role raised the abort flag.
__device__ __forceinline__ bool tc_wait(uint32_t bar, uint32_t parity, volatile uint32_t* abort_flag,
                                        uint32_t* flags, uint64_t timeout_ns = kWaitTimeoutNs) {
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if ((it & 63u) == 0 && global_timer_ns() - t0 > timeout_ns) {
            *abort_flag = 1u;
            if (flags) atomicOr(flags, kFlagTimeout);
            return false;
        }
    }
}

// Self-test of the bounded waits, on mbarriers that nothing ever completes (no copy,
// no MMA, no fault): thread 0 waits with a short limit and must give up, record the
// timeout flag and raise the abort flag; thread 32 waits with the kernels' full limit and
// must give up early through that abort flag.  out[0..3]: thread 0 gave up, thread 32 gave
// up, thread 32's wait in microseconds, the flag word.
__global__ void __launch_bounds__(64) wait_selftest_kernel(uint32_t* out, uint64_t short_ns) {
    __shared__ __align__(8) uint64_t bars[2];
    __shared__ uint32_t abort_word;
    if (threadIdx.x == 0) {
        mbar_init(smem_u32(&bars[0]), 1);
        mbar_init(smem_u32(&bars[1]), 1);
        abort_word = 0u;
        fence_mbar_init();
    }
    __syncthreads();
    volatile uint32_t* abort_flag = &abort_word;
    if (threadIdx.x == 0) {
        const bool done = tc_wait(smem_u32(&bars[0]), 0u, abort_flag, out + 3, short_ns);
        out[0] = done ? 0u : 1u;
    } else if (threadIdx.x == 32) {
        const uint64_t t0 = global_timer_ns();
        const bool done = tc_wait(smem_u32(&bars[1]), 0u, abort_flag, nullptr);
        out[2] = static_cast<uint32_t>((global_timer_ns() - t0) / 1000u);
        out[1] = done ? 0u : 1u;
    }
}

template <int D>
__global__ void __launch_bounds__(TcShape<D>::kThreads, 1)
    prefill_tc_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ CUtensorMap kmap,
                      const __grid_constant__ CUtensorMap vmap) {
    using T = TcShape<D>;
    constexpr int M = T::kM, N = T::kN, ST = T::kStages;
    using O = OperandGeom<D>;  // staging of Q, K and V: O::kBlk blocks of [rows][O::kCols]
    constexpr int kGroups = N / 32; // 32-token boxes per tile
    constexpr uint32_t kIdescQK = bf16_idesc(M, N, false);
    constexpr uint32_t kIdescPV = bf16_idesc(M, D, true);
    // mbarrier indices
    constexpr int kQFull = 0, kKFull = 1, kKEmpty = 1 + ST, kVFull = 1 + 2 * ST, kVEmpty = 1 + 3 * ST;
    constexpr int kSFull = 1 + 4 * ST, kSFree = 3 + 4 * ST, kPFull = 5 + 4 * ST, kPVDone = 6 + 4 * ST;
    constexpr int kDrain = 7 + 4 * ST, kXchg = 8 + 4 * ST, kBars = 12 + 4 * ST;  // kXchg: one per lane quadrant
    constexpr int SW = T::kSoftmaxThreads;
    static_assert(8 * kBars + 8 <= 512, "barrier area");
    static_assert(512 + 3 * 2 * M * 4 <= T::kHeaderBytes, "header");

    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t bar0 = smem_u32(smem);
    auto bar = [bar0](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 8 * kBars);
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + 8 * kBars + 4);
    float* xmax = reinterpret_cast<float*>(smem + 512);  // [tile parity][half][row] partial row maxima
    float* xsum = xmax + 2 * 2 * M;                       // [half][row] partial row sums
    const uint32_t tb = (bar0 + T::kHeaderBytes + 1023u) & ~1023u;  // tiles, 1024-byte aligned
    const uint32_t q_s = tb + T::kQOff, p_s = tb + T::kPOff;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // ---- work item: (sequence b, kv head, block of M query rows)
    const int rb = blockIdx.x % p.blocks_per_head;
    const int bh = blockIdx.x / p.blocks_per_head;
    const int kvh = bh % p.Hkv;
    const int b = bh / p.Hkv;
    const int R = p.Lq * p.g;
    const int row0 = rb * M;

    if (threadIdx.x == 0) {
        mbar_init(bar(kQFull), SW);
#pragma unroll
        for (int s = 0; s < ST; ++s) {
            mbar_init(bar(kKFull + s), 1);
            mbar_init(bar(kKEmpty + s), 1);
            mbar_init(bar(kVFull + s), 1);
            mbar_init(bar(kVEmpty + s), 1);
        }
        mbar_init(bar(kSFull), 1);
        mbar_init(bar(kSFull + 1), 1);
        mbar_init(bar(kSFree), SW);
        mbar_init(bar(kSFree + 1), SW);
        mbar_init(bar(kPFull), SW);
#pragma unroll
        for (int qd = 0; qd < 4; ++qd) mbar_init(bar(kXchg + qd), 64);
        mbar_init(bar(kPVDone), 1);
        mbar_init(bar(kDrain), 1);
        *abort_flag = 0u;
        fence_mbar_init();
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
    }
    if (warp == T::kMmaWarp) {
        tc_alloc(smem_u32(tmem_slot), T::kTmemCols);
        tc_relinquish();
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
    const int i_last = min(p.Lq - 1, (min(row0 + M, R) - 1) / p.g);
    int kv_end = L;  // keys this block can see: [0, kv_end)
    if (p.causal_offset >= 0) kv_end = max(0, min(L, p.causal_offset + i_last + 1));
    const int ntiles = (kv_end + N - 1) / N;

    tc_fence_before();
    __syncthreads();  // barriers initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_launch_dependents();

    bool ok = true;
    if (warp == T::kProducerWarp) {
        // ================= producer: TMA loads of the K and V tiles
        const uint64_t pol = l2_policy_evict_last();  // the other row blocks of this head read the same tiles
        constexpr int kTB = 32 / kGroups;             // tiles whose pages one warp-wide load resolves
        int32_t pg = 0;
        int k_issued = 0, v_issued = 0;
        for (int j = 0; j < ntiles; ++j) {
            if (j % kTB == 0) {
                const int jj = j + lane / kGroups;
                const int t0 = jj * N + (lane % kGroups) * 32;
                pg = 0;
                if (jj < ntiles && t0 < kv_end) {
                    pg = p.page_table == nullptr
                             ? b
                             : __ldcg(p.page_table + static_cast<int64_t>(b) * p.pt_s0 +
                                      static_cast<int64_t>(t0 / p.P) * p.pt_s1);
                }
            }
            int32_t pages[kGroups];
#pragma unroll
            for (int q = 0; q < kGroups; ++q) pages[q] = __shfl_sync(0xffffffffu, pg, (j % kTB) * kGroups + q);
            const int ng = min(kGroups, (kv_end - j * N + 31) / 32);  // boxes of this tile holding visible keys
            const uint32_t bytes = static_cast<uint32_t>(ng) * 32u * D * 2u;
            const int stage = j % ST;
            const uint32_t par = static_cast<uint32_t>((j / ST) - 1) & 1u;
#pragma unroll
            for (int kv = 0; kv < 2; ++kv) {
                if (j >= ST) ok = tc_wait(bar((kv ? kVEmpty : kKEmpty) + stage), par, abort_flag, p.flags);
                ok = __all_sync(0xffffffffu, ok);
                if (!ok) break;
                if (lane == 0) {
                    const uint32_t full = bar((kv ? kVFull : kKFull) + stage);
                    const uint32_t dst = tb + (kv ? T::kVOff : T::kKOff) + static_cast<uint32_t>(stage) * T::kKVBytes;
                    mbar_arrive_expect_tx(full, bytes);
#pragma unroll
                    for (int q = 0; q < kGroups; ++q) {
                        if (q >= ng) break;
                        const int page = pages[q];
                        if ((page < 0 || page >= p.NP) && p.flags) atomicOr(p.flags, kFlagPageOOR);
                        const int slot = (j * N + 32 * q) % p.P;
                        if constexpr (D == 32) {
                            tma_load_4d(dst + static_cast<uint32_t>(q * 32 * O::kRowBytes), kv ? &vmap : &kmap, full,
                                        0, kvh, slot, page, pol);
                        } else {
#pragma unroll
                            for (int c = 0; c < O::kBlk; ++c)
                                tma_load_5d(dst + static_cast<uint32_t>(c * N * O::kRowBytes + q * 32 * O::kRowBytes),
                                            kv ? &vmap : &kmap, full, 0, kvh, slot, page, c, pol);
                        }
                    }
                }
                __syncwarp();
                if (kv) v_issued = j + 1; else k_issued = j + 1;
            }
            if (!ok) break;
        }
        if (!ok && lane == 0) {
            // wait (bounded) for the copies still in flight before the CTA can exit
            for (int s = 0; s < ST; ++s) {
                if (k_issued > s) {
                    const int jl = s + ST * ((k_issued - 1 - s) / ST);
                    mbar_wait_bounded(bar(kKFull + s), static_cast<uint32_t>(jl / ST) & 1u, kWaitTimeoutNs);
                }
                if (v_issued > s) {
                    const int jl = s + ST * ((v_issued - 1 - s) / ST);
                    mbar_wait_bounded(bar(kVFull + s), static_cast<uint32_t>(jl / ST) & 1u, kWaitTimeoutNs);
                }
            }
        }
    } else if (warp == T::kMmaWarp) {
        // ================= MMA issuer (one thread)
        if (lane == 0 && ntiles > 0) {
            bool issued = false;
            // O += P_jj V_jj, K = N keys in steps of 16
            auto pv = [&](int jj) -> bool {
                if (!tc_wait(bar(kPFull), static_cast<uint32_t>(jj) & 1u, abort_flag, p.flags)) return false;
                if (!tc_wait(bar(kVFull + jj % ST), static_cast<uint32_t>(jj / ST) & 1u, abort_flag, p.flags))
                    return false;
                tc_fence_after();
                const uint32_t vb = tb + T::kVOff + static_cast<uint32_t>(jj % ST) * T::kKVBytes;
#pragma unroll
                for (int k = 0; k < N / 16; ++k) {
                    const uint32_t po = static_cast<uint32_t>((k >> 2) * (M * 128) + (k & 3) * 32);
                    tc_mma_bf16(tmem + T::kColO, sw128_desc(p_s + po, 16, 1024),
                                O::desc(vb + static_cast<uint32_t>(k * 16 * O::kRowBytes), N * O::kRowBytes), kIdescPV,
                                (jj > 0 || k > 0) ? 1u : 0u);
                }
                tc_commit(bar(kPVDone));
                tc_commit(bar(kVEmpty + jj % ST));
                return true;
            };
            ok = tc_wait(bar(kQFull), 0, abort_flag, p.flags);
            for (int j = 0; ok && j < ntiles; ++j) {
                const int stage = j % ST;
                ok = tc_wait(bar(kKFull + stage), static_cast<uint32_t>(j / ST) & 1u, abort_flag, p.flags);
                if (ok && j >= 2) ok = tc_wait(bar(kSFree + (j & 1)), static_cast<uint32_t>((j - 2) >> 1) & 1u,
                                               abort_flag, p.flags);
                if (!ok) break;
                tc_fence_after();
                // S_j = Q K_j^T, K = D in steps of 16
                const uint32_t kb = tb + T::kKOff + static_cast<uint32_t>(stage) * T::kKVBytes;
                const uint32_t d = tmem + T::kColS + static_cast<uint32_t>((j & 1) * N);
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    tc_mma_bf16(d, O::desc(q_s + O::kstep(k, M), 16), O::desc(kb + O::kstep(k, N), 16), kIdescQK,
                                k > 0 ? 1u : 0u);
                }
                tc_commit(bar(kSFull + (j & 1)));
                tc_commit(bar(kKEmpty + stage));
                issued = true;
                if (j >= 1) ok = pv(j - 1);
            }
            if (ok) ok = pv(ntiles - 1);
            if (!ok && issued) {
                // wait (bounded) for the MMAs still in flight
                tc_commit(bar(kDrain));
                mbar_wait_bounded(bar(kDrain), 0, kWaitTimeoutNs);
            }
        }
    } else {
        // ================= softmax warps: warps w and w + 4 share TMEM lane quadrant w
        // (rows 32w .. 32w + 31, one per thread) and take half of each row's columns
        // O columns per warp: half of them each, or (D = 32, one 32-column load) all of
        // them for the first half and none for the second
        constexpr int NH = N / 2, DH = D >= 64 ? D / 2 : D;
        const int quad = warp & 3, h = warp >> 2;
        const bool o_owner = D >= 64 || h == 0;
        const int r = 32 * quad + lane;
        const int cb = h * NH;  // this warp's first column of S (and key of the tile)
        const uint32_t t_lane = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t xbar = bar(kXchg + quad);
        stage_q_tile<D>(q_s, p, b, kvh, row0, R, threadIdx.x, SW);
        fence_proxy_async_smem();
        mbar_arrive(bar(kQFull));

        const int rg = row0 + r;
        const bool row_ok = rg < R;
        const int qi = row_ok ? rg / p.g : 0;
        const int qh = kvh * p.g + (row_ok ? rg - qi * p.g : 0);
        int lim = row_ok ? L : 0;  // the row sees keys t < lim (and the mask)
        if (p.causal_offset >= 0) lim = min(lim, p.causal_offset + qi + 1);
        const uint8_t* mrow = p.mask ? p.mask + b * p.m_sb + static_cast<int64_t>(qi) * p.m_si : nullptr;
        // exponent = fma(s, cs, -reference): the scale is folded into the FFMA when it is
        // positive (then max(s) * cs is the scaled maximum); otherwise S is pre-scaled
        const bool prescale = !(p.scale_log2 > 0.f);
        const float cs = prescale ? 1.f : p.scale_log2;
        float m_used = -INFINITY;  // reference maximum of the row's exponentials (log2 domain)
        float l = 0.f;             // this half's share of the row sum
        for (int j = 0; j < ntiles; ++j) {
            const int sb = j & 1;
            __syncwarp();  // the tcgen05 loads below are warp-collective
            ok = __all_sync(0xffffffffu, tc_wait(bar(kSFull + sb), static_cast<uint32_t>(j >> 1) & 1u, abort_flag,
                                                 p.flags));
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[NH];
#pragma unroll
            for (int c = 0; c < NH / 32; ++c)
                tc_ld32(tmem + t_lane + T::kColS + static_cast<uint32_t>(sb * N + cb + 32 * c),
                        *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
            tc_wait_ld();
            tc_fence_before();
            mbar_arrive(bar(kSFree + sb));  // S buffer may take tile j + 2

            // ---- visibility (invisible -> -inf) and this half's maximum (8 chains)
            const int t0 = j * N + cb;
            if (prescale) {
#pragma unroll
                for (int c = 0; c < NH; ++c) sr[c] = __float_as_uint(__uint_as_float(sr[c]) * p.scale_log2);
            }
            if (!(t0 + NH <= lim && !mrow)) {
#pragma unroll
                for (int c = 0; c < NH; ++c) {
                    const int t = t0 + c;
                    bool vis = t < lim;
                    if (vis && mrow) vis = mrow[static_cast<int64_t>(t) * p.m_st] != 0;
                    if (!vis) sr[c] = __float_as_uint(-INFINITY);
                }
            }
            float mx[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) mx[e] = __uint_as_float(sr[e]);
#pragma unroll
            for (int c = 8; c < NH; c += 16) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    mx[e] = fmax3(mx[e], __uint_as_float(sr[c + e]), __uint_as_float(sr[c + 8 + e < NH ? c + 8 + e : c + e]));
            }
            const float mr = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7]));
            // ---- the row's maximum over both halves (exchange phase j of this quadrant)
            xmax[((j & 1) * 2 + h) * M + r] = mr;
            mbar_arrive(xbar);
            ok = __all_sync(0xffffffffu, tc_wait(xbar, static_cast<uint32_t>(j) & 1u, abort_flag, p.flags));
            if (!ok) break;
            const float mt = fmaxf(mr, xmax[((j & 1) * 2 + (h ^ 1)) * M + r]) * cs;
            // ---- lazy rescale decision: move the reference only when the maximum grows
            // by more than 2^8 (both halves of a row decide alike from the same values)
            float alpha = 1.f;
            bool grow = false;
            if (m_used == -INFINITY) {
                m_used = mt;  // O is still exactly zero for this row
            } else if (mt > m_used + 8.f) {
                grow = true;
                alpha = ex2_approx(m_used - mt);
                m_used = mt;
            }
            // ---- P = 2^(s * cs - reference) into registers while P_{j-1} V_{j-1} runs
            const float nref = (m_used == -INFINITY) ? 0.f : -m_used;
            uint32_t pw[NH / 2];
            const uint64_t cs2 = f2_pack(cs, cs), nref2 = f2_pack(nref, nref);
            uint64_t rs2[2] = {0ull, 0ull};
#pragma unroll
            for (int c = 0; c < NH / 2; ++c) {
                const uint64_t x2 =
                    f2_fma(f2_pack(__uint_as_float(sr[2 * c]), __uint_as_float(sr[2 * c + 1])), cs2, nref2);
                float x0, x1;
                f2_unpack(x2, x0, x1);
                const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                rs2[c & 1] = f2_add(rs2[c & 1], f2_pack(p0, p1));
                pw[c] = pack_bf16x2(p0, p1);
            }
            float ra, rb;
            f2_unpack(f2_add(rs2[0], rs2[1]), ra, rb);
            l = l * alpha + (ra + rb);
            // ---- O and the P buffer are free once P_{j-1} V_{j-1} has completed
            if (j > 0) {
                ok = __all_sync(0xffffffffu, tc_wait(bar(kPVDone), static_cast<uint32_t>(j - 1) & 1u, abort_flag,
                                                     p.flags));
                if (!ok) break;
                tc_fence_after();
            }
            if (o_owner && __any_sync(0xffffffffu, grow)) {
#pragma unroll 1
                for (int c = 0; c < DH / 32; ++c) {  // this warp's O columns
                    uint32_t o[32];
                    const uint32_t ta = tmem + t_lane + T::kColO + static_cast<uint32_t>(h * DH + 32 * c);
                    tc_ld32(ta, o);
                    tc_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tc_st32(ta, o);
                }
                tc_wait_st();
            }
            // ---- P (bf16) into the swizzled K-major A layout
#pragma unroll
            for (int c8 = 0; c8 < NH / 8; ++c8) {
                const int cc = cb / 8 + c8;  // 16-byte chunk of the row in the tile
                st_shared_v4(p_s + static_cast<uint32_t>((cc >> 3) * (M * 128) + r * 128 + (((cc & 7) ^ (r & 7)) << 4)),
                             pw[4 * c8], pw[4 * c8 + 1], pw[4 * c8 + 2], pw[4 * c8 + 3]);
            }
            // ---- last tile: V rows past the last visible key hold anything (NaN
            // included, or nothing loaded): zero them before they meet a zero weight
            if (j == ntiles - 1 && j * N + N > kv_end) {
                const int stage = j % ST;
                ok = __all_sync(0xffffffffu, tc_wait(bar(kVFull + stage), static_cast<uint32_t>(j / ST) & 1u,
                                                     abort_flag, p.flags));
                if (!ok) break;
                const int v0 = kv_end - j * N;
                const uint32_t vb = tb + T::kVOff + static_cast<uint32_t>(stage) * T::kKVBytes;
                zero_v_rows<D, N>(vb, v0, threadIdx.x, SW);
            }
            fence_proxy_async_smem();  // P (and the zeroed V rows) -> tensor core
            tc_fence_before();
            mbar_arrive(bar(kPFull));
        }
        // ---- epilogue: out = O / l (zeros for a row that saw no key); each warp
        // stores its half of the row's columns
        if (ok && ntiles > 0) {
            ok = __all_sync(0xffffffffu, tc_wait(bar(kPVDone), static_cast<uint32_t>(ntiles - 1) & 1u, abort_flag,
                                                 p.flags));
            if (ok) tc_fence_after();
        }
        if (ok) {  // the row sum over both halves (exchange phase ntiles)
            xsum[h * M + r] = l;
            mbar_arrive(xbar);
            ok = __all_sync(0xffffffffu, tc_wait(xbar, static_cast<uint32_t>(ntiles) & 1u, abort_flag, p.flags));
        }
        __syncwarp();
        if (ok) {
            const float lt = l + xsum[(h ^ 1) * M + r];
            const float inv = lt > 0.f ? 1.f / lt : 0.f;
            if (o_owner)
                store_o_row<DH>(tmem + t_lane + T::kColO + static_cast<uint32_t>(h * DH), ntiles > 0, inv, row_ok,
                                p.out + b * p.o_sb + qi * p.o_si + qh * p.o_sh + h * DH);
        }
    }
    // ---- all roles meet before the TMEM columns are freed
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == T::kMmaWarp) {
        tc_fence_after();
        tc_dealloc(tmem, T::kTmemCols);
    }
}


// ======================================================================
// Two Q tiles per CTA (D = 64, 128): 256 query rows share every K/V tile.
//
//  * Warps 0-3 own Q tile 0 (rows 0-127), warps 4-7 Q tile 1 (rows 128-255), one
//    full row per thread; warp 8 is the producer, warp 9 lane 0 the MMA issuer.
//  * TMEM: S_t (t = 0, 1) at columns 128 t, N = 128 fp32 columns each; P_t (bf16
//    pairs, 64 columns) is written over the first half of S_t once S_t has been
//    read; O_t at 256 + D t.  S_t = Q_t K^T takes A and B from shared memory;
//    O_t += P_t V takes A (P_t) from TMEM and B (V) from shared memory.
//  * The issuer alternates the two tiles (Q_0K_j, Q_1K_j, P_0V_j, Q_0K_{j+1},
//    P_1V_j, Q_1K_{j+1}, ...), so each softmax warpgroup works on its S while the
//    tensor core serves the other.  Tensor-core operations of one thread run in
//    issue order and a commit covers every earlier one, so S_t(j) being full also
//    means P_t(j-1) V_{j-1} has finished: O_t may be rescaled and P_t rewritten
//    without a further wait.
//  * K and V tiles share one ring of kSlots slots (K_j is load 2j, V_j load 2j+1).
// ======================================================================
__device__ __forceinline__ void tc_mma_bf16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

template <int D>
struct Tc2Shape {
    static constexpr int kM = 128;  // rows per Q tile (TMEM lanes); two tiles per CTA
    static constexpr int kN = 128;  // keys per tile
    static constexpr int kSlots = (D == 32) ? 16 : (D == 64) ? 8 : 4;
    static constexpr int kThreads = 320;  // warps 0-7 softmax, 8 producer, 9 MMA issuer
    static constexpr int kProducerWarp = 8, kMmaWarp = 9;
    static constexpr uint32_t kQBytes = kM * D * 2;  // one Q tile
    static constexpr uint32_t kSlotBytes = kN * D * 2;
    static constexpr uint32_t kQOff = 0;
    static constexpr uint32_t kRingOff = 2 * kQBytes;
    static constexpr uint32_t kTileBytes = kRingOff + kSlots * kSlotBytes;
    static constexpr uint32_t kHeaderBytes = 1024;
    static constexpr uint32_t kSmemBytes = kHeaderBytes + 1024 + kTileBytes;
    static constexpr uint32_t kTmemCols = 512;
    static constexpr uint32_t kColS = 0;    // S_t at 128 t
    static constexpr uint32_t kColO = 256;  // O_t at 256 + D t
    static_assert(D == 32 || D == 64 || D == 128, "two-tile kernel: D = 32, 64 or 128");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kSmemBytes > 232448 / 2, "one CTA per SM, so the 512 TMEM columns are always free");
};

template <int D>
__global__ void __launch_bounds__(Tc2Shape<D>::kThreads, 1)
    prefill_tc2_kernel(const __grid_constant__ PrefillParams p, const __grid_constant__ CUtensorMap kmap,
                       const __grid_constant__ CUtensorMap vmap) {
    using T = Tc2Shape<D>;
    constexpr int M = T::kM, N = T::kN, NS = T::kSlots;
    using O = OperandGeom<D>;
    constexpr int kGroups = N / 32;
    constexpr uint32_t kIdescQK = bf16_idesc(M, N, false);
    constexpr uint32_t kIdescPV = bf16_idesc(M, D, true);
    // mbarrier indices
    // P full per (Q tile t, key part h): index kParts t + h (P is handed over N / kParts keys at a time)
    constexpr int kParts = APD_PREFILL_P_PARTS;
    static_assert(kParts == 1 || kParts == 2 || kParts == 4, "P hand-over parts");
    constexpr int kQFull = 0, kFull = 1, kEmpty = 1 + NS, kSFull = 1 + 2 * NS, kPFull = 3 + 2 * NS;
    constexpr int kPVDone = kPFull + 2 * kParts, kDrain = kPVDone + 2, kBars = kDrain + 1;
    static_assert(8 * kBars + 8 <= T::kHeaderBytes, "header");

    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t bar0 = smem_u32(smem);
    auto bar = [bar0](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 8 * kBars);
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + 8 * kBars + 4);
    const uint32_t tb = (bar0 + T::kHeaderBytes + 1023u) & ~1023u;  // tiles, 1024-byte aligned
    const uint32_t ring = tb + T::kRingOff;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int rb = blockIdx.x % p.blocks_per_head;
    const int bh = blockIdx.x / p.blocks_per_head;
    const int kvh = bh % p.Hkv;
    const int b = bh / p.Hkv;
    const int R = p.Lq * p.g;
    const int row0 = rb * 2 * M;

    if (threadIdx.x == 0) {
        mbar_init(bar(kQFull), 256);
#pragma unroll
        for (int s = 0; s < NS; ++s) {
            mbar_init(bar(kFull + s), 1);
            mbar_init(bar(kEmpty + s), 1);
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar(kSFull + t), 1);
#pragma unroll
            for (int h = 0; h < kParts; ++h) mbar_init(bar(kPFull + kParts * t + h), 128);
            mbar_init(bar(kPVDone + t), 1);
        }
        mbar_init(bar(kDrain), 1);
        *abort_flag = 0u;
        fence_mbar_init();
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
    }
    if (warp == T::kMmaWarp) {
        tc_alloc(smem_u32(tmem_slot), T::kTmemCols);
        tc_relinquish();
    }
    pdl_wait_prior_grid();

    const int64_t cap = static_cast<int64_t>(p.MP) * p.P;
    int L = __ldcg(p.seq_lens + b);
    if (L < 0 || L > cap) {
        if (p.flags && threadIdx.x == 0) atomicOr(p.flags, L < 0 ? kFlagLenNegative : kFlagLenClamped);
        L = L < 0 ? 0 : static_cast<int>(cap);
    }
    const int i_last = min(p.Lq - 1, (min(row0 + 2 * M, R) - 1) / p.g);
    int kv_end = L;
    if (p.causal_offset >= 0) kv_end = max(0, min(L, p.causal_offset + i_last + 1));
    const int ntiles = (kv_end + N - 1) / N;

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_launch_dependents();

    bool ok = true;
    if (warp == T::kProducerWarp) {
        // ================= producer: K_j and V_j tiles through the shared ring
        const uint64_t pol = l2_policy_evict_last();
        constexpr int kTB = 32 / kGroups;
        int32_t pg = 0;
        int issued = 0;
        for (int n = 0; n < 2 * ntiles; ++n) {
            const int j = n >> 1, kv = n & 1;
            if (kv == 0 && j % kTB == 0) {
                const int jj = j + lane / kGroups;
                const int t0 = jj * N + (lane % kGroups) * 32;
                pg = 0;
                if (jj < ntiles && t0 < kv_end) {
                    pg = p.page_table == nullptr
                             ? b
                             : __ldcg(p.page_table + static_cast<int64_t>(b) * p.pt_s0 +
                                      static_cast<int64_t>(t0 / p.P) * p.pt_s1);
                }
            }
            int32_t pages[kGroups];
#pragma unroll
            for (int q = 0; q < kGroups; ++q) pages[q] = __shfl_sync(0xffffffffu, pg, (j % kTB) * kGroups + q);
            const int ng = min(kGroups, (kv_end - j * N + 31) / 32);
            const int slot = n % NS;
            if (n >= NS) ok = tc_wait(bar(kEmpty + slot), static_cast<uint32_t>((n / NS) - 1) & 1u, abort_flag, p.flags);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (lane == 0) {
                const uint32_t full = bar(kFull + slot);
                const uint32_t dst = ring + static_cast<uint32_t>(slot) * T::kSlotBytes;
                mbar_arrive_expect_tx(full, static_cast<uint32_t>(ng) * 32u * D * 2u);
#pragma unroll
                for (int q = 0; q < kGroups; ++q) {
                    if (q >= ng) break;
                    const int page = pages[q];
                    if ((page < 0 || page >= p.NP) && p.flags) atomicOr(p.flags, kFlagPageOOR);
                    const int sl = (j * N + 32 * q) % p.P;
                    if constexpr (D == 32) {
                        tma_load_4d(dst + static_cast<uint32_t>(q * 32 * O::kRowBytes), kv ? &vmap : &kmap, full, 0,
                                    kvh, sl, page, pol);
                    } else {
#pragma unroll
                        for (int c = 0; c < O::kBlk; ++c)
                            tma_load_5d(dst + static_cast<uint32_t>(c * N * O::kRowBytes + q * 32 * O::kRowBytes),
                                        kv ? &vmap : &kmap, full, 0, kvh, sl, page, c, pol);
                    }
                }
            }
            __syncwarp();
            issued = n + 1;
        }
        if (!ok && lane == 0) {
            for (int s = 0; s < NS; ++s) {
                if (issued > s) {
                    const int nl = s + NS * ((issued - 1 - s) / NS);
                    mbar_wait_bounded(bar(kFull + s), static_cast<uint32_t>(nl / NS) & 1u, kWaitTimeoutNs);
                }
            }
        }
    } else if (warp == T::kMmaWarp) {
        // ================= MMA issuer (one thread)
        if (lane == 0 && ntiles > 0) {
            bool issued = false;
            auto wait_load = [&](int n) {
                return tc_wait(bar(kFull + n % NS), static_cast<uint32_t>(n / NS) & 1u, abort_flag, p.flags);
            };
            // S_t = Q_t K_j^T
            auto qk = [&](int t, int j) {
                const uint32_t kb = ring + static_cast<uint32_t>((2 * j) % NS) * T::kSlotBytes;
                const uint32_t qb = tb + static_cast<uint32_t>(t) * T::kQBytes;
#pragma unroll
                for (int k = 0; k < D / 16; ++k) {
                    tc_mma_bf16(tmem + T::kColS + 128u * t, O::desc(qb + O::kstep(k, M), 16), O::desc(kb + O::kstep(k, N), 16),
                                kIdescQK, k > 0 ? 1u : 0u);
                }
                tc_commit(bar(kSFull + t));
            };
            // O_t += P_t V_j over part h of the keys, P_t from TMEM (8 columns per 16 keys)
            auto pv = [&](int t, int j, int h) {
                const uint32_t vb = ring + static_cast<uint32_t>((2 * j + 1) % NS) * T::kSlotBytes;
#pragma unroll
                for (int kk = 0; kk < N / 16 / kParts; ++kk) {
                    const int k = (N / 16 / kParts) * h + kk;
                    tc_mma_bf16_ts(tmem + T::kColO + static_cast<uint32_t>(D * t), tmem + T::kColS + 128u * t + 8u * k,
                                   O::desc(vb + static_cast<uint32_t>(k * 16 * O::kRowBytes), N * O::kRowBytes), kIdescPV,
                                   (j > 0 || k > 0) ? 1u : 0u);
                }
                if (h == kParts - 1) tc_commit(bar(kPVDone + t));
            };
            // the parts of P_t(j) V_j, each as soon as the softmax warpgroup hands it over
            auto pv_halves = [&](int t, int j) -> bool {
#pragma unroll
                for (int h = 0; h < kParts; ++h) {
                    if (!tc_wait(bar(kPFull + kParts * t + h), static_cast<uint32_t>(j) & 1u, abort_flag, p.flags))
                        return false;
                    tc_fence_after();
                    pv(t, j, h);
                }
                return true;
            };
            ok = tc_wait(bar(kQFull), 0, abort_flag, p.flags) && wait_load(0);
            if (ok) {
                tc_fence_after();
                qk(0, 0);
                qk(1, 0);
                tc_commit(bar(kEmpty + 0));
                issued = true;
            }
            for (int j = 0; ok && j < ntiles; ++j) {
                ok = wait_load(2 * j + 1) && pv_halves(0, j);
                if (!ok) break;
                if (j + 1 < ntiles) {
                    ok = wait_load(2 * j + 2);
                    if (!ok) break;
                    tc_fence_after();
                    qk(0, j + 1);
                }
                ok = pv_halves(1, j);
                if (!ok) break;
                tc_commit(bar(kEmpty + (2 * j + 1) % NS));  // V_j read by both tiles
                if (j + 1 < ntiles) {
                    qk(1, j + 1);
                    tc_commit(bar(kEmpty + (2 * j + 2) % NS));  // K_{j+1} read by both tiles
                }
            }
            if (!ok && issued) {
                tc_commit(bar(kDrain));
                mbar_wait_bounded(bar(kDrain), 0, kWaitTimeoutNs);
            }
        }
    } else {
        // ================= softmax warpgroup t: thread = one full row of Q tile t
        const int t = warp >> 2, quad = warp & 3;
        const int r = 32 * quad + lane;
        const int wt = threadIdx.x & 127;
        const uint32_t t_lane = static_cast<uint32_t>(quad * 32) << 16;
        const uint32_t s_col = T::kColS + 128u * t;
        const uint32_t o_col = T::kColO + static_cast<uint32_t>(D * t);
        const uint32_t q_s = tb + static_cast<uint32_t>(t) * T::kQBytes;
        stage_q_tile<D>(q_s, p, b, kvh, row0 + M * t, R, wt, 128);
        fence_proxy_async_smem();
        mbar_arrive(bar(kQFull));

        const int rg = row0 + M * t + r;
        const bool row_ok = rg < R;
        const int qi = row_ok ? rg / p.g : 0;
        const int qh = kvh * p.g + (row_ok ? rg - qi * p.g : 0);
        int lim = row_ok ? L : 0;
        if (p.causal_offset >= 0) lim = min(lim, p.causal_offset + qi + 1);
        const uint8_t* mrow = p.mask ? p.mask + b * p.m_sb + static_cast<int64_t>(qi) * p.m_si : nullptr;
        const bool prescale = !(p.scale_log2 > 0.f);
        const float cs = prescale ? 1.f : p.scale_log2;
        float m_used = -INFINITY, l = 0.f;
        for (int j = 0; j < ntiles; ++j) {
            __syncwarp();
            ok = __all_sync(0xffffffffu, tc_wait(bar(kSFull + t), static_cast<uint32_t>(j) & 1u, abort_flag, p.flags));
            if (!ok) break;
            tc_fence_after();
            uint32_t sr[N];
#pragma unroll
            for (int c = 0; c < N / 32; ++c)
                tc_ld32(tmem + t_lane + s_col + static_cast<uint32_t>(32 * c),
                        *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
            tc_wait_ld();
            // ---- visibility (invisible -> -inf) and the row maximum (8 chains)
            const int t0 = j * N;
            if (prescale) {
#pragma unroll
                for (int c = 0; c < N; ++c) sr[c] = __float_as_uint(__uint_as_float(sr[c]) * p.scale_log2);
            }
            if (!(t0 + N <= lim && !mrow)) {
#pragma unroll
                for (int c = 0; c < N; ++c) {
                    const int tk = t0 + c;
                    bool vis = tk < lim;
                    if (vis && mrow) vis = mrow[static_cast<int64_t>(tk) * p.m_st] != 0;
                    if (!vis) sr[c] = __float_as_uint(-INFINITY);
                }
            }
            float mx[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) mx[e] = __uint_as_float(sr[e]);
#pragma unroll
            for (int c = 8; c < N; c += 16) {
#pragma unroll
                for (int e = 0; e < 8; ++e)
                    mx[e] = fmax3(mx[e], __uint_as_float(sr[c + e]), __uint_as_float(sr[c + 8 + e < N ? c + 8 + e : c + e]));
            }
            const float mt = fmax3(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5]), fmaxf(mx[6], mx[7])) * cs;
            // ---- lazy rescale (S_t(j) full implies P_t(j-1) V_{j-1} has finished)
            float alpha = 1.f;
            bool grow = false;
            if (m_used == -INFINITY) {
                m_used = mt;
            } else if (mt > m_used + 8.f) {
                grow = true;
                alpha = ex2_approx(m_used - mt);
                m_used = mt;
            }
            if (__any_sync(0xffffffffu, grow)) {
#pragma unroll 1
                for (int c = 0; c < D / 32; ++c) {
                    uint32_t o[32];
                    const uint32_t ta = tmem + t_lane + o_col + static_cast<uint32_t>(32 * c);
                    tc_ld32(ta, o);
                    tc_wait_ld();
#pragma unroll
                    for (int e = 0; e < 32; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
                    tc_st32(ta, o);
                }
            }
            // ---- last tile: V rows past the last visible key hold anything (NaN
            // included, or nothing loaded): tile 0's warpgroup zeroes them before
            // either tile multiplies them by a zero weight
            if (t == 0 && j == ntiles - 1 && j * N + N > kv_end) {
                const int nv = 2 * j + 1;
                ok = __all_sync(0xffffffffu, tc_wait(bar(kFull + nv % NS), static_cast<uint32_t>(nv / NS) & 1u,
                                                     abort_flag, p.flags));
                if (!ok) break;
                const int v0 = kv_end - j * N;
                const uint32_t vb = ring + static_cast<uint32_t>(nv % NS) * T::kSlotBytes;
                zero_v_rows<D, N>(vb, v0, wt, 128);
                fence_proxy_async_smem();  // before the first half of P is handed over
            }
            // ---- P = 2^(s * cs - reference) as bf16 pairs over the first half of S_t,
            // handed to the MMA issuer N / kParts keys at a time
            const float nref = (m_used == -INFINITY) ? 0.f : -m_used;
            const uint64_t cs2 = f2_pack(cs, cs), nref2 = f2_pack(nref, nref);
            uint64_t rs2[2] = {0ull, 0ull};
#pragma unroll
            for (int hh = 0; hh < N / 32; ++hh) {  // 32 keys -> 16 TMEM columns of bf16 pairs
                uint32_t pw[16];
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    const uint64_t x2 = f2_fma(
                        f2_pack(__uint_as_float(sr[32 * hh + 2 * c]), __uint_as_float(sr[32 * hh + 2 * c + 1])), cs2,
                        nref2);
                    float x0, x1;
                    f2_unpack(x2, x0, x1);
                    const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
                    rs2[c & 1] = f2_add(rs2[c & 1], f2_pack(p0, p1));
                    pw[c] = pack_bf16x2(p0, p1);
                }
                tc_st16(tmem + t_lane + s_col + static_cast<uint32_t>(16 * hh), pw);
                constexpr int kPer = (N / 32) / kParts;  // 32-key chunks per part
                if (hh % kPer == kPer - 1) {
                    tc_wait_st();
                    tc_fence_before();
                    mbar_arrive(bar(kPFull + kParts * t + hh / kPer));
                }
            }
            float ra, rb;
            f2_unpack(f2_add(rs2[0], rs2[1]), ra, rb);
            l = l * alpha + (ra + rb);

        }
        // ---- epilogue: out = O_t / l (zeros for a row that saw no key)
        if (ok && ntiles > 0) {
            ok = __all_sync(0xffffffffu, tc_wait(bar(kPVDone + t), static_cast<uint32_t>(ntiles - 1) & 1u, abort_flag,
                                                 p.flags));
            if (ok) tc_fence_after();
        }
        __syncwarp();
        if (ok) {
            // a row that saw no visible key outputs zeros (its emulated exponentials of
            // -inf are tiny, not 0, so test the running maximum rather than l)
            const float inv = (l > 0.f && m_used != -INFINITY) ? 1.f / l : 0.f;
            store_o_row<D>(tmem + t_lane + o_col, ntiles > 0, inv, row_ok, p.out + b * p.o_sb + qi * p.o_si + qh * p.o_sh);
        }
    }
    // ---- all roles meet before the TMEM columns are freed
    __syncwarp();
    tc_fence_before();
    __syncthreads();
    if (warp == T::kMmaWarp) {
        tc_fence_after();
        tc_dealloc(tmem, T::kTmemCols);
    }
}

}  // namespace apd
