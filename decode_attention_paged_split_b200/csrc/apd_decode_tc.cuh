// apd_decode_tc.cuh -- decode attention for kv heads shared by more than 16 query heads, on
// the sm_100a fifth-generation tensor cores (tcgen05 + TMEM).
//
// Same operation as the split kernel (AstrAI commit log of csrc/kernels/attn_paged_decode.cu:
// one query token per sequence, paged bf16 K/V, split-KV partials o_part / ml_part merged by
// one combine kernel); this is the design for kv heads whose query heads fill a tensor-core
// tile.  With g = 32 query heads per kv head, every K/V tile meets 32 query rows, twice the
// 16 of one mma.sync head block; here the tile goes to the tensor core once for all of them.
// The heads are padded to NH = 32 or 64 with zero Q rows, whose outputs are never written.
// Above 64 query heads per kv head the heads are cut into nhb = ceil(g / 64) blocks of
// equal size rounded up to 16 heads (g = 80: 48 + 32), one CTA per block and split.  The
// blocks' CTAs of one split read the same K/V tiles; when they run at the same time (the
// automatic split count keeps every CTA in one wave) the later reads are L2 hits.
//
//  - A CTA owns one split of one (sequence b, kv head, q-head block) unit: a contiguous run
//    of the sequence's 32-token boxes, cut exactly as the fixed-split plan cuts it.  With at most
//    8 splits per unit the splits of a unit form one thread-block cluster: each split leaves
//    its unnormalised part in its own shared memory, and split c then merges heads c, c + nk,
//    c + 2 nk, ... of all nk parts over distributed shared memory and writes them out (one
//    kernel, no partials in global memory).  With more splits the parts go to the
//    fixed-split slots of o_part / ml_part and the combine kernel merges them.
//  - Tokens are the M side of both products, query heads the N side:
//      S^T[t][h]  = sum_d K[t][d] Q[h][d]        (M = 128 tokens, N = NH heads, K = D;
//                                                 A = the K tile, B = Q, both K-major)
//      O^T[d][h] += sum_t V[t][d] P^T[t][h]      (M = D, N = NH heads, K = 128 tokens;
//                                                 A = the V tile read MN-major, B = P^T
//                                                 MN-major: P stored [token][head])
//    so the staged K and V tiles are used exactly as the TMA lands them.
//  - Two producer warps (after the softmax warps) resolve each tile's four pages and issue
//    the TMA loads of its K boxes and its V boxes into two rings, each refilled as soon as
//    its own stage is free: a K stage right after its S^T product, a V stage after its P V.
//    One lane of the warp between them issues the MMAs, each product as soon as its operands
//    are ready (S^T_j does not wait for P_{j-1} V_{j-1}, nor that for the next K tile), and
//    commits them to the mbarriers that free the stages and hand S^T to the softmax warps.
//    Two S^T buffers (and at 32 heads two P buffers) let the softmax of tile j + 1 run while
//    P_j V_j is on the tensor core.
//  - Softmax warps, one group of 4 per 32 heads (warps 0-3, and 4-7 at 64 heads): TMEM lane t
//    is token t of the tile, so thread t of a group reads its token's 32 scores of the
//    group's heads with one tcgen05.ld and owns those exponentials.  The reference maximum
//    of each head is shared by all tokens (in shared memory); it moves only when some score
//    exceeds it by more than 2^8 (one OR-vote per tile and group over the group's named
//    barrier; the head maxima are then reduced across its 128 threads, O^T and the running
//    sums rescaled).  Each thread keeps its own running sums of the bf16 weights it wrote;
//    they are added across the threads once, at the end.
//
// Every mbarrier wait is bounded.  A wait that runs out raises a shared abort flag that every
// role polls; the softmax warps decide to stop only through the result of a barrier
// reduction, so the warps of a group leave together, and all warps meet before the TMEM
// columns are freed and, with the cluster merge, at the cluster barrier.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cstdint>

#include "apd_kernels.cuh"
#include "apd_prefill_tc.cuh"
#include "apd_ptx.cuh"

namespace apd {

struct McParams {
    const __nv_bfloat16* q;  // [B][Hq][D], head dim contiguous
    int64_t q_sb, q_sh;
    const int32_t* page_table;  // NULL: contiguous KV, sequence b is page b of P tokens
    int64_t pt_s0, pt_s1;
    const int32_t* seq_lens;
    __nv_bfloat16* out;
    int64_t out_sb, out_sh;
    float* o_part;   // [slots][rows_max][D]
    float* ml_part;  // [slots][rows_max][2]
    uint32_t* flags;
    int32_t B, Hkv, g, HB, rows_max, P, NP, MP;
    int32_t nhb, hbh; // q-head blocks per kv head, q heads per block (a multiple of 16, <= NH)
    int32_t ksplit;   // splits per (sequence, kv head, q-head block)
    int32_t cluster;  // 1: the ksplit CTAs of a unit are one cluster and merge over DSMEM
    float scale_log2;
    uint64_t wait_ns;         // limit of each wait (kWaitTimeoutNs; shorter in the self-test)
    int32_t test_skip_pfull;  // self-test only: the softmax warps never hand over P of tile 1
};

// Instruction descriptor of tcgen05.mma kind::f16: bf16 A and B, fp32 D, each operand
// K-major or MN-major (bits 15 and 16), shape M x N.
constexpr uint32_t mc_idesc(int M, int N, bool a_mn_major, bool b_mn_major) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
           (static_cast<uint32_t>(N >> 3) << 17) | (static_cast<uint32_t>(M >> 4) << 24);
}

// OR of `pred` over the `nthreads` threads that meet at named barrier `id` (every warp of
// them arrives with all its lanes).
__device__ __forceinline__ bool bar_any(int id, int nthreads, bool pred) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
        : "memory");
    return r != 0u;
}
__device__ __forceinline__ void bar_named(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Reduce-scatter of 32 values over the warp: afterwards v[0] of lane t holds the
// reduction over the 32 lanes of value t (recursive halving: at offset o, a lane keeps the
// upper half of its values when bit o of its lane index is set and takes the partner's
// copy of them).
template <bool kMax>
__device__ __forceinline__ void warp_reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
        const bool upper = (lane & o) != 0;
#pragma unroll
        for (int i = 0; i < o; ++i) {
            const float keep = upper ? v[i + o] : v[i];
            const float send = upper ? v[i] : v[i + o];
            const float got = __shfl_xor_sync(0xffffffffu, send, o);
            v[i] = kMax ? fmaxf(keep, got) : keep + got;
        }
    }
}

// ---- thread-block cluster pieces: the cluster barrier, DSMEM addressing and loads, and
// mbarrier arrivals and waits across the cluster
__device__ __forceinline__ void cluster_arrive_relaxed() {
    asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
// The address in CTA `rank` of the cluster of this CTA's shared-memory address `addr`.
__device__ __forceinline__ uint32_t dsmem_addr(uint32_t addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}
// The generic address of the same variable in CTA `rank` of the cluster (plain loads
// through it read that CTA's shared memory).
template <typename T>
__device__ __forceinline__ const T* dsmem_ptr(const T* p, uint32_t rank) {
    uint64_t r;
    asm("mapa.u64 %0, %1, %2;" : "=l"(r) : "l"(reinterpret_cast<uint64_t>(p)), "r"(rank));
    return reinterpret_cast<const T*>(r);
}
__device__ __forceinline__ void fence_acq_rel_cluster() { asm volatile("fence.acq_rel.cluster;" ::: "memory"); }
// Arrive on an mbarrier of another CTA of the cluster (address from dsmem_addr), releasing
// this thread's earlier writes at cluster scope.
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_bar) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint32_t bar, uint32_t parity) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(bar), "r"(parity)
        : "memory");
    return done != 0;
}
// warp_wait with acquire at cluster scope (for arrivals from other CTAs of the cluster).
__device__ __forceinline__ bool warp_wait_cluster(uint32_t bar, uint32_t parity, uint64_t timeout_ns,
                                                  volatile uint32_t* abort_word, uint32_t* flags) {
    bool done = mbar_try_wait_acq_cluster(bar, parity);
    if (__all_sync(0xffffffffu, done)) return true;
    const uint64_t t0 = global_timer_ns();
    for (uint32_t it = 1;; ++it) {
        if (!done) done = mbar_try_wait_acq_cluster(bar, parity);
        if (__all_sync(0xffffffffu, done)) return true;
        if ((it & 15u) == 0) {
            int give_up = 0;
            if ((threadIdx.x & 31) == 0 && global_timer_ns() - t0 > timeout_ns) give_up = 1;
            give_up = __shfl_sync(0xffffffffu, give_up, 0);
            if (give_up) {
                if ((threadIdx.x & 31) == 0) {
                    *abort_word = 1u;
                    atomicOr(flags, kFlagTimeout);
                }
                return false;
            }
        }
    }
}

constexpr int kMcMaxCluster = 8;  // splits per unit merged over DSMEM (the portable cluster size)

template <int D, int NH>
struct McShape {
    static_assert(D == 128 && (NH == 32 || NH == 64), "the tensor-core decode kernel: D = 128, 32 or 64 heads");
    static constexpr int kTok = 128;  // tokens per tile (TMEM lanes of S^T)
    static constexpr int kGroups = NH / 32;  // softmax groups of 4 warps, 32 heads each
    // K and V ring depths: 3 + 3 stages of 32 KB.  At 64 heads Q and P double, and the third
    // K stage fits only with one P buffer (the 2-stage K ring bounded the tile period there:
    // traced 1.38 us against 1.18 us at 32 heads)
    static constexpr int kKStages = 3, kVStages = 3;
    static constexpr int kPBuffers = NH == 32 ? 2 : 1;
    static constexpr int kSoftmaxWarps = 4 * kGroups;
    static constexpr int kProducerWarp = kSoftmaxWarps, kMmaWarp = kSoftmaxWarps + 1,
                         kVProducerWarp = kSoftmaxWarps + 2;
    static constexpr int kThreads = 32 * (kSoftmaxWarps + 3);
    static constexpr uint32_t kQBytes = NH * D * 2;
    static constexpr uint32_t kKVBytes = kTok * D * 2;  // one K (or V) tile
    static constexpr uint32_t kPBytes = kTok * NH * 2;
    static constexpr uint32_t kQOff = 0;
    static constexpr uint32_t kKOff = kQBytes;
    static constexpr uint32_t kVOff = kKOff + kKStages * kKVBytes;
    static constexpr uint32_t kPOff = kVOff + kVStages * kKVBytes;
    static constexpr uint32_t kTileBytes = kPOff + kPBuffers * kPBytes;
    // header (mbarriers, TMEM address, abort flag, the per-warp head maxima and the reference
    // maxima), up to 1 KB to reach 1024-byte alignment, then the tiles.  The per-warp head
    // sums of the epilogue go to the second half of the Q buffer, idle by then.
    static constexpr uint32_t kHeaderBytes = NH == 32 ? 2048 : 1792;
    static constexpr uint32_t kRedOff = 512;
    static constexpr uint32_t kSmemBytes = kHeaderBytes + 1024 + kTileBytes;
    static constexpr uint32_t kTmemCols = NH == 32 ? 128 : 256;
    static constexpr uint32_t kColS = 0;        // two S^T buffers: columns [0, 2 NH)
    static constexpr uint32_t kColO = 2 * NH;   // O^T: columns [2 NH, 3 NH)
    static_assert(kColO + NH <= kTmemCols, "TMEM columns");
    // cluster merge: a split's part [NH][D] fp32 + [NH][2] in its K ring, its merge weights
    // [kMcMaxCluster + 1][NH] in its Q buffer
    static_assert(NH * D * 4 + NH * 8 <= kKStages * kKVBytes, "part in the K ring");
    static_assert((kMcMaxCluster + 1) * NH * 4 <= kQBytes, "merge weights in the Q buffer");
    static_assert(kRedOff + kGroups * 4 * 32 * 4 + NH * 4 <= kHeaderBytes, "header");
    static_assert(4 * NH * 4 <= kQBytes / 2 && (kMcMaxCluster + 1) * NH * 4 <= kQBytes / 2,
                  "epilogue sums and merge weights in the two halves of the Q buffer");
    static_assert(kSmemBytes <= 232448, "shared memory per CTA");
    static_assert(kSmemBytes > 232448 / 2, "one CTA per SM, so the TMEM columns are always free");
};

template <int D, int NH>
__global__ void __launch_bounds__(McShape<D, NH>::kThreads, 1)
    decode_mq_tc_kernel(const __grid_constant__ McParams p, const __grid_constant__ CUtensorMap kmap,
                        const __grid_constant__ CUtensorMap vmap) {
    using T = McShape<D, NH>;
    using O = OperandGeom<D>;   // K, V and Q staging: D/64 blocks of [rows][64]
    using PG = OperandGeom<NH>; // P staging: [tokens][NH] rows of 2 NH bytes
    constexpr int TK = T::kTok, KST = T::kKStages, VST = T::kVStages, NG = T::kGroups;
    constexpr uint32_t kIdescQK = mc_idesc(TK, NH, false, false);
    constexpr uint32_t kIdescPV = mc_idesc(D, NH, true, true);
    // mbarriers; S, P and PVDone come in pairs, one per S / P buffer (tile parity)
    constexpr int kQFull = 0, kKFull = 1, kKEmpty = 1 + KST, kVFull = 1 + 2 * KST, kVEmpty = 1 + 2 * KST + VST;
    constexpr int kSFull = 1 + 2 * (KST + VST), kSFree = kSFull + 2, kPFull = kSFull + 4, kPVDone = kSFull + 6;
    constexpr int kDrain = kSFull + 8, kParts = kSFull + 9, kBars = kSFull + 10;
    constexpr int kSoftThreads = 32 * T::kSoftmaxWarps;
    // named barriers: 1 + g for the 4 warps of softmax group g, kAllBarId for all of them
    constexpr int kAllBarId = 1 + NG;
    static_assert(8 * kBars + 8 <= static_cast<int>(T::kRedOff), "barrier area");

    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t bar0 = smem_u32(smem);
    auto bar = [bar0](int i) { return bar0 + 8u * static_cast<uint32_t>(i); };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + 8 * kBars);
    volatile uint32_t* abort_flag = reinterpret_cast<volatile uint32_t*>(smem + 8 * kBars + 4);
    float* s_red = reinterpret_cast<float*>(smem + T::kRedOff);  // [group][4 warps][32] head maxima
    float* s_m = s_red + NG * 4 * 32;                             // [NH] the heads' reference maxima
    const uint32_t tb = (bar0 + T::kHeaderBytes + 1023u) & ~1023u;
    // [4 warps][NH] head sums, written in the epilogue once every S^T product is done
    float* s_sum = reinterpret_cast<float*>(smem + (tb + T::kQOff + T::kQBytes / 2 - bar0));
    const uint32_t q_s = tb + T::kQOff, p_s = tb + T::kPOff;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    // ---- work item: split `split` of q-head block hb of unit (sequence b, kv head kvh); the
    // block holds q heads h0 .. h0 + gh - 1 of the kv head's g
    const int nsplit = p.ksplit;
    const int ub = blockIdx.x / nsplit;
    const int split = blockIdx.x - ub * nsplit;
    const int u2 = ub / p.nhb;
    const int hb = ub - u2 * p.nhb;
    const int b = u2 / p.Hkv;
    const int kvh = u2 - b * p.Hkv;
    const int h0 = hb * p.hbh;
    const int gh = min(p.hbh, p.g - h0);
    const int qh0 = kvh * p.g + h0;  // first q head of the block

    if (threadIdx.x == 0) {
        mbar_init(bar(kQFull), kSoftThreads);
#pragma unroll
        for (int s = 0; s < KST; ++s) {
            mbar_init(bar(kKFull + s), 1);
            mbar_init(bar(kKEmpty + s), 1);
        }
#pragma unroll
        for (int s = 0; s < VST; ++s) {
            mbar_init(bar(kVFull + s), 1);
            mbar_init(bar(kVEmpty + s), 1);
        }
        mbar_init(bar(kSFull), 1);
        mbar_init(bar(kSFull + 1), 1);
        mbar_init(bar(kSFree), kSoftThreads);
        mbar_init(bar(kSFree + 1), kSoftThreads);
        mbar_init(bar(kPFull), kSoftThreads);
        mbar_init(bar(kPFull + 1), kSoftThreads);
        mbar_init(bar(kPVDone), 1);
        mbar_init(bar(kPVDone + 1), 1);
        mbar_init(bar(kDrain), 1);
        mbar_init(bar(kParts), static_cast<uint32_t>(max(1, nsplit - 1)));  // one arrival per other split
        *abort_flag = 0u;
        fence_mbar_init();
        prefetch_tensormap(&kmap);
        prefetch_tensormap(&vmap);
    }
    __syncthreads();
    // cluster phase 0 (waited before any DSMEM access): every CTA has initialised its mbarriers
    if (p.cluster) cluster_arrive_relaxed();
    // Launched with programmatic dependent launch: nothing above reads global memory.
    pdl_wait_prior_grid();
    pdl_launch_dependents();

    // ---- the sequence's length and this split's boxes [c0, c1) of 32 tokens, cut as the
    // fixed-split plan cuts them (the combine recomputes the same cut)
    const bool contig = p.page_table == nullptr;
    const int64_t cap = static_cast<int64_t>(p.MP) * p.P;
    int L = __ldcg(p.seq_lens + b);
    if (L < 0 || L > cap) {
        if (threadIdx.x == 0 && split == 0 && hb == 0)
            atomicOr(p.flags, L < 0 ? kFlagLenNegative : kFlagLenClamped);
        L = L < 0 ? 0 : static_cast<int>(cap);
    }
    const int n32 = (L + kTile - 1) / kTile;
    int c0 = 0, c1 = 0, nk = 1;
    if (n32 > 0) {
        const int S = max(1, min(nsplit, n32));
        const int c = (n32 + S - 1) / S;
        c0 = min(split * c, n32);
        c1 = min(c0 + c, n32);
        nk = (n32 + c - 1) / c;
    }
    if (c0 >= c1) {
        // an empty split writes nothing; split 0 of an empty sequence writes its zero rows
        if (split == 0) {
            for (int i = threadIdx.x; i < gh * (D / 8); i += blockDim.x) {
                const int h = i / (D / 8), ch = i - h * (D / 8);
                *reinterpret_cast<uint4*>(p.out + b * p.out_sb + static_cast<int64_t>(qh0 + h) * p.out_sh +
                                          8 * ch) = make_uint4(0u, 0u, 0u, 0u);
            }
        }
        if (p.cluster) {
            cluster_wait();
            if (threadIdx.x < nsplit && threadIdx.x != split) mbar_arrive_remote(dsmem_addr(bar(kParts), threadIdx.x));
            cluster_arrive();
            cluster_wait();
        }
        return;  // the whole CTA, before any TMEM allocation or copy
    }
    const int tok0 = kTile * c0;
    const int tok1 = min(kTile * c1, L);
    const int ntiles = (tok1 - tok0 + TK - 1) / TK;

    if (warp == T::kMmaWarp) {
        tc_alloc(smem_u32(tmem_slot), T::kTmemCols);
        tc_relinquish();
    }
    tc_fence_before();
    __syncthreads();  // TMEM allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    bool ok = true;
    bool cluster_waited = false;  // this thread has waited for cluster phase 0
    if (warp == T::kProducerWarp || warp == T::kVProducerWarp) {
        // ================= producers: TMA loads of the K tiles or the V tiles, four 32-token
        // boxes each
        const int kv = warp == T::kVProducerWarp ? 1 : 0;
        const CUtensorMap* map = kv ? &vmap : &kmap;
        const int full0 = kv ? kVFull : kKFull, empty0 = kv ? kVEmpty : kKEmpty;
        const int ST = kv ? VST : KST;
        const uint32_t ring = tb + (kv ? T::kVOff : T::kKOff);
        // every K/V byte leaves HBM once: one CTA reads it, or the blocks' CTAs of one split
        // read it about together (measured at g = 80: DRAM reads = the algorithmic bytes)
        const uint64_t pol = l2_policy_evict_first();
        constexpr int kBoxes = TK / kTile;               // 4
        constexpr int kTB = 32 / kBoxes;                 // tiles whose pages one warp-wide load resolves
        int32_t pg = 0;
        int issued = 0;
        for (int j = 0; j < ntiles; ++j) {
            if (j % kTB == 0) {
                const int jj = j + lane / kBoxes;
                const int t = tok0 + jj * TK + (lane % kBoxes) * kTile;
                pg = 0;
                if (jj < ntiles && t < tok1)
                    pg = contig ? b
                                : __ldcg(p.page_table + static_cast<int64_t>(b) * p.pt_s0 +
                                         static_cast<int64_t>(t / p.P) * p.pt_s1);
            }
            int32_t pages[kBoxes];
#pragma unroll
            for (int q = 0; q < kBoxes; ++q) pages[q] = __shfl_sync(0xffffffffu, pg, (j % kTB) * kBoxes + q);
            const int ng = min(kBoxes, (tok1 - (tok0 + j * TK) + kTile - 1) / kTile);  // boxes holding tokens
            const uint32_t bytes = static_cast<uint32_t>(ng) * kTile * D * 2u;
            const int stage = j % ST;
            if (j >= ST) ok = tc_wait(bar(empty0 + stage), static_cast<uint32_t>((j / ST) - 1) & 1u, abort_flag, p.flags, p.wait_ns);
            ok = __all_sync(0xffffffffu, ok);
            if (!ok) break;
            if (lane == 0) {
                const uint32_t full = bar(full0 + stage);
                const uint32_t dst = ring + static_cast<uint32_t>(stage) * T::kKVBytes;
                mbar_arrive_expect_tx(full, bytes);
#pragma unroll
                for (int q = 0; q < kBoxes; ++q) {
                    if (q >= ng) break;
                    const int page = pages[q];
                    if (kv == 0 && (page < 0 || page >= p.NP)) atomicOr(p.flags, kFlagPageOOR);
                    const int tok = tok0 + j * TK + kTile * q;
                    const int slot = contig ? tok : tok % p.P;
#pragma unroll
                    for (int c = 0; c < O::kBlk; ++c)
                        tma_load_5d(dst + static_cast<uint32_t>(c * TK * O::kRowBytes + q * kTile * O::kRowBytes), map,
                                    full, 0, kvh, slot, page, c, pol);
                }
            }
            __syncwarp();
            issued = j + 1;
        }
        if (!ok && lane == 0) {
            // wait (bounded) for the copies still in flight before the CTA can exit
            for (int s = 0; s < ST; ++s) {
                if (issued > s) {
                    const int jl = s + ST * ((issued - 1 - s) / ST);
                    mbar_wait_bounded(bar(full0 + s), static_cast<uint32_t>(jl / ST) & 1u, p.wait_ns);
                }
            }
        }
    } else if (warp == T::kMmaWarp) {
        // ================= MMA issuer (one thread): S^T_jq as soon as K_jq is staged and its
        // S buffer is free, P_jp V_jp as soon as P_jp and V_jp are; tcgen05 operations of one
        // thread run in issue order, so the P V products accumulate into O^T in tile order
        if (lane == 0) {
            bool issued = false;
            ok = tc_wait(bar(kQFull), 0, abort_flag, p.flags, p.wait_ns);
            int jq = 0, jp = 0;
            uint64_t t_idle = global_timer_ns();
            for (uint32_t it = 1; ok && jp < ntiles; ++it) {
                bool progress = false;
                if (jq < ntiles && mbar_try_wait(bar(kKFull + jq % KST), static_cast<uint32_t>(jq / KST) & 1u) &&
                    (jq < 2 || mbar_try_wait(bar(kSFree + (jq & 1)), static_cast<uint32_t>((jq - 2) >> 1) & 1u))) {
                    tc_fence_after();
                    // S^T_jq = K_jq Q^T, K = D in steps of 16
                    const uint32_t kb = tb + T::kKOff + static_cast<uint32_t>(jq % KST) * T::kKVBytes;
                    const uint32_t d = tmem + T::kColS + static_cast<uint32_t>((jq & 1) * NH);
#pragma unroll
                    for (int k = 0; k < D / 16; ++k)
                        tc_mma_bf16(d, O::desc(kb + O::kstep(k, TK), 16), O::desc(q_s + O::kstep(k, NH), 16),
                                    kIdescQK, k > 0 ? 1u : 0u);
                    tc_commit(bar(kSFull + (jq & 1)));
                    tc_commit(bar(kKEmpty + jq % KST));
                    issued = true;
                    progress = true;
                    ++jq;
                }
                if (jp < jq && mbar_try_wait(bar(kPFull + (jp & 1)), static_cast<uint32_t>(jp >> 1) & 1u) &&
                    mbar_try_wait(bar(kVFull + jp % VST), static_cast<uint32_t>(jp / VST) & 1u)) {
                    tc_fence_after();
                    // O^T += V_jp^T P_jp^T, K = TK tokens in steps of 16
                    const uint32_t vb = tb + T::kVOff + static_cast<uint32_t>(jp % VST) * T::kKVBytes;
                    const uint32_t pb = p_s + static_cast<uint32_t>((jp % T::kPBuffers) * T::kPBytes);
#pragma unroll
                    for (int k = 0; k < TK / 16; ++k)
                        tc_mma_bf16(tmem + T::kColO,
                                    O::desc(vb + static_cast<uint32_t>(k * 16 * O::kRowBytes), TK * O::kRowBytes),
                                    PG::desc(pb + static_cast<uint32_t>(k * 16 * PG::kRowBytes), TK * PG::kRowBytes),
                                    kIdescPV, (jp > 0 || k > 0) ? 1u : 0u);
                    tc_commit(bar(kPVDone + (jp & 1)));
                    tc_commit(bar(kVEmpty + jp % VST));
                    progress = true;
                    ++jp;
                }
                if (progress) {
                    it = 0;
                } else if (*abort_flag) {
                    ok = false;
                } else if ((it & 63u) == 0) {
                    const uint64_t now = global_timer_ns();
                    if (it == 64) t_idle = now;  // the first check of an idle stretch starts its clock
                    else if (now - t_idle > p.wait_ns) {
                        *abort_flag = 1u;
                        atomicOr(p.flags, kFlagTimeout);
                        ok = false;
                    }
                }
            }
            if (!ok && issued) {
                // wait (bounded) for the MMAs still in flight
                tc_commit(bar(kDrain));
                mbar_wait_bounded(bar(kDrain), 0, p.wait_ns);
            }
        }
    } else {
        // ================= softmax warps: group grp (warps 4 grp .. 4 grp + 3) owns heads
        // [32 grp, 32 grp + 32); thread r of a group owns token r of each tile (TMEM lane r)
        const int grp = warp >> 2, wq = warp & 3;
        const int r = 32 * wq + lane;
        const int hoff = 32 * grp;
        const int gbar = 1 + grp;  // this group's named barrier
        const uint32_t t_lane = static_cast<uint32_t>(32 * wq) << 16;
        // Q rows kvh * g + h0 + h (h < NH) in the K-major B layout [D/64][NH][64]; rows at
        // and past gh (padding up to NH) are zeros.  A thread's loads are all issued before
        // its stores.
        {
            constexpr int kPer = NH * (D / 8) / kSoftThreads;  // 16-byte chunks per thread
            static_assert(NH * (D / 8) % kSoftThreads == 0, "Q chunks per thread");
            uint4 v[kPer];
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int idx = threadIdx.x + u * kSoftThreads;
                const int h = idx / (D / 8), ch = idx - h * (D / 8);
                v[u] = h < gh ? __ldg(reinterpret_cast<const uint4*>(
                                    p.q + b * p.q_sb + static_cast<int64_t>(qh0 + h) * p.q_sh + 8 * ch))
                              : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int u = 0; u < kPer; ++u) {
                const int idx = threadIdx.x + u * kSoftThreads;
                const int h = idx / (D / 8), ch = idx - h * (D / 8);
                st_shared_v4(q_s + static_cast<uint32_t>((ch / O::kChunks) * (NH * O::kRowBytes) + h * O::kRowBytes +
                                                         (O::swz(h, ch % O::kChunks) << 4)),
                             v[u].x, v[u].y, v[u].z, v[u].w);
            }
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(kQFull));

        // the reference maximum of each of the group's heads (log2 domain) lives in shared
        // memory (the same for every thread of the group; written only when it moves)
        float* const g_m = s_m + hoff;
        if (wq == 0) g_m[lane] = -INFINITY;
        bar_named(gbar, 128);
        auto load_m = [&](float (&mv)[32]) {
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 a = *reinterpret_cast<const float4*>(g_m + i);
                mv[i] = a.x;
                mv[i + 1] = a.y;
                mv[i + 2] = a.z;
                mv[i + 3] = a.w;
            }
        };
        float l[32];  // this thread's sums of the bf16 weights, relative to the reference
#pragma unroll
        for (int i = 0; i < 32; ++i) l[i] = 0.f;
        float* const g_red = s_red + grp * 4 * 32;  // this group's [4 warps][32] maxima
        bool wok = true, stopped = false;
        for (int j = 0; j < ntiles; ++j) {
            const int sb = j & 1;
            float x[32];
            wok = warp_wait(bar(kSFull + sb), static_cast<uint32_t>(j >> 1) & 1u, p.wait_ns, abort_flag,
                            p.flags);
            if (wok) {
                uint32_t sr[32];
                tc_fence_after();
                tc_ld32(tmem + t_lane + T::kColS + static_cast<uint32_t>(sb * NH + hoff), sr);
                tc_wait_ld();
                tc_fence_before();
                mbar_arrive(bar(kSFree + sb));  // the S buffer may take tile j + 2
                const bool valid = tok0 + j * TK + r < tok1;
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = valid ? __uint_as_float(sr[i]) * p.scale_log2 : -INFINITY;
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) x[i] = -INFINITY;
            }
            bool need = false;
            {
                float m[32];
                load_m(m);
#pragma unroll
                for (int i = 0; i < 32; ++i) need |= x[i] > m[i] + 8.f;
            }
            // one vote per tile and group: a new reference for some head, or some warp gave up
            const bool gave_up = !wok || *abort_flag != 0u;
            if (bar_any(gbar, 128, need || gave_up)) {
                if (bar_any(gbar, 128, gave_up)) {
                    stopped = true;
                    break;
                }
                // ---- new reference: the tile's maximum of each head over the 128 tokens
                float v[32];
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = x[i];
                warp_reduce_scatter32<true>(v, lane);
                g_red[wq * 32 + lane] = v[0];
                bar_named(gbar, 128);
                float alpha[32];
                float mnew = 0.f;  // lane i: the new reference of head i
                {
                    float m[32];
                    load_m(m);
#pragma unroll
                    for (int i = 0; i < 32; i += 4) {
                        float4 a = *reinterpret_cast<const float4*>(g_red + i);
#pragma unroll
                        for (int w = 1; w < 4; ++w) {
                            const float4 q = *reinterpret_cast<const float4*>(g_red + w * 32 + i);
                            a.x = fmaxf(a.x, q.x);
                            a.y = fmaxf(a.y, q.y);
                            a.z = fmaxf(a.z, q.z);
                            a.w = fmaxf(a.w, q.w);
                        }
                        const float tm[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
                        for (int e = 0; e < 4; ++e) {
                            const float mn = fmaxf(m[i + e], tm[e]);
                            // 1 for a head whose maximum did not move; 0 while m is -inf
                            alpha[i + e] = (mn == m[i + e]) ? 1.f : ex2_approx(m[i + e] - mn);
                            if (lane == i + e) mnew = mn;
                            l[i + e] *= alpha[i + e];
                        }
                    }
                }
                bar_named(gbar, 128);  // every thread has read the old references
                if (wq == 0) g_m[lane] = mnew;
                bar_named(gbar, 128);  // the new references are visible to the group
                if (j > 0) {
                    // O^T holds P V of the earlier tiles: rescale this thread's row (head dim
                    // r) in the group's columns once the last P V has landed (in issue order,
                    // so every earlier one has too)
                    wok = warp_wait(bar(kPVDone + ((j - 1) & 1)), static_cast<uint32_t>((j - 1) >> 1) & 1u,
                                    p.wait_ns, abort_flag, p.flags);
                    if (wok) {
                        tc_fence_after();
                        uint32_t o[32];
                        const uint32_t oa = tmem + t_lane + T::kColO + static_cast<uint32_t>(hoff);
                        tc_ld32(oa, o);
                        tc_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha[i]);
                        tc_st32(oa, o);
                        tc_wait_st();
                    }
                }
            }
            if (!wok) continue;  // gave up in this tile: the next vote stops every warp of the group

            // ---- P = 2^(x - m) as bf16 pairs, and the sums of exactly those weights
            uint32_t pw[16];
#pragma unroll
            for (int i = 0; i < 16; i += 2) {
                const float4 mv = *reinterpret_cast<const float4*>(g_m + 2 * i);
                const float m4[4] = {mv.x, mv.y, mv.z, mv.w};
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const float p0 = ex2_approx(x[2 * (i + e)] - m4[2 * e]);
                    const float p1 = ex2_approx(x[2 * (i + e) + 1] - m4[2 * e + 1]);
                    pw[i + e] = pack_bf16x2(p0, p1);
                    l[2 * (i + e)] += bf16_lo(pw[i + e]);
                    l[2 * (i + e) + 1] += bf16_hi(pw[i + e]);
                }
            }
            // ---- the P buffer of tile j is free once P V of the tile before that used it has
            // completed: j - 2 with two buffers, j - 1 with one
            {
                constexpr int kBack = T::kPBuffers;
                if (j >= kBack) {
                    const int jb = j - kBack;
                    wok = warp_wait(bar(kPVDone + (jb & 1)), static_cast<uint32_t>(jb >> 1) & 1u, p.wait_ns,
                                    abort_flag, p.flags);
                    if (!wok) continue;
                    tc_fence_after();
                }
            }
            // the group's 64 bytes of row r of P^T ([token][head], 2 NH bytes, swizzled as the
            // MN-major B layout)
            const uint32_t pb = p_s + static_cast<uint32_t>((j % T::kPBuffers) * T::kPBytes);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                st_shared_v4(pb + static_cast<uint32_t>(r * PG::kRowBytes + (PG::swz(r, 4 * grp + q) << 4)),
                             pw[4 * q], pw[4 * q + 1], pw[4 * q + 2], pw[4 * q + 3]);
            // ---- last tile: V rows past the split's last token hold anything (NaN included,
            // or nothing loaded): zero them before they meet a zero weight
            if (j == ntiles - 1 && tok0 + j * TK + TK > tok1) {
                const int stage = j % VST;
                wok = warp_wait(bar(kVFull + stage), static_cast<uint32_t>(j / VST) & 1u, p.wait_ns, abort_flag,
                                p.flags);
                if (!wok) continue;
                zero_v_rows<D, TK>(tb + T::kVOff + static_cast<uint32_t>(stage) * T::kKVBytes, tok1 - (tok0 + j * TK),
                                   threadIdx.x, kSoftThreads);
            }
            fence_proxy_async_smem();  // P (and the zeroed V rows) -> tensor core
            tc_fence_before();
            if (!(p.test_skip_pfull && j == 1)) mbar_arrive(bar(kPFull + (j & 1)));
        }
        // ---- epilogue: the heads' sums over the CTA's tokens, then out (or the partial, or the
        // cluster part).  Heads at and past g are padding (zero Q rows): never written.
        if (!stopped && wok)
            wok = warp_wait(bar(kPVDone + ((ntiles - 1) & 1)), static_cast<uint32_t>((ntiles - 1) >> 1) & 1u,
                            p.wait_ns, abort_flag, p.flags);
        {
            float v[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = l[i];
            warp_reduce_scatter32<false>(v, lane);
            s_sum[wq * NH + hoff + lane] = v[0];
        }
        const bool gave_up = stopped || !wok || *abort_flag != 0u;
        const bool any_gave_up = bar_any(gbar, 128, gave_up);
        const int dd = r;  // this thread's head-dim column of O (TMEM lane of O^T)
        uint32_t o[32];
        float lt[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
            o[i] = 0u;
            lt[i] = 0.f;
        }
        if (!any_gave_up) {
            tc_fence_after();
            tc_ld32(tmem + t_lane + T::kColO + static_cast<uint32_t>(hoff), o);
            tc_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                float4 a = *reinterpret_cast<const float4*>(s_sum + hoff + i);
#pragma unroll
                for (int w = 1; w < 4; ++w) {
                    const float4 q = *reinterpret_cast<const float4*>(s_sum + w * NH + hoff + i);
                    a.x += q.x;
                    a.y += q.y;
                    a.z += q.z;
                    a.w += q.w;
                }
                lt[i] = a.x;
                lt[i + 1] = a.y;
                lt[i + 2] = a.z;
                lt[i + 3] = a.w;
            }
        }
        // m and l of the group's head `lane`, for the writes of (m, l) pairs
        const float mm = g_m[lane];
        float ll = 0.f;
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (lane == i) ll = lt[i];
        if (nk == 1) {
            // the only non-empty split: normalised rows straight to out
            if (!any_gave_up) {
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int h = hoff + i;
                    if (h < gh)
                        p.out[b * p.out_sb + static_cast<int64_t>(qh0 + h) * p.out_sh + dd] =
                            __float2bfloat16_rn(__uint_as_float(o[i]) / lt[i]);
                }
            }
        } else if (!p.cluster) {
            if (!any_gave_up) {
                // the partial of this split, for each block of 16 q heads (h0 is a multiple of
                // 16): slot ((b * Hkv + kvh) * HB + hh / 16) * ksplit + split, row hh % 16 of
                // q head hh = h0 + h of the kv head
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int h = h0 + hoff + i;
                    if (hoff + i < gh) {
                        const int64_t slot = (static_cast<int64_t>(u2) * p.HB + h / kMaxRows) * p.ksplit + split;
                        p.o_part[(slot * p.rows_max + h % kMaxRows) * D + dd] = __uint_as_float(o[i]);
                    }
                }
                if (wq == 0 && hoff + lane < gh) {
                    const int h = h0 + hoff + lane;
                    const int64_t slot = (static_cast<int64_t>(u2) * p.HB + h / kMaxRows) * p.ksplit + split;
                    *reinterpret_cast<float2*>(p.ml_part + (slot * p.rows_max + h % kMaxRows) * 2) =
                        make_float2(mm, ll);
                }
            }
        } else {
            // ---- merge over the cluster.  Part of split s: [NH][D] fp32 (O^T unnormalised),
            // then [NH] (m, l) pairs, at the start of its K ring (free once its last S^T is done)
            float* const part_p = reinterpret_cast<float*>(smem + (tb + T::kKOff - bar0));
            cluster_wait();  // phase 0: every CTA of the cluster has its mbarriers initialised
            cluster_waited = true;
#pragma unroll
            for (int i = 0; i < 32; ++i) part_p[(hoff + i) * D + dd] = __uint_as_float(o[i]);
            if (wq == 0) {
                part_p[NH * D + 2 * (hoff + lane)] = mm;
                part_p[NH * D + 2 * (hoff + lane) + 1] = ll;
            }
            fence_acq_rel_cluster();
            bar_named(kAllBarId, kSoftThreads);  // both groups' halves of the part are written
            // tell every other CTA of the cluster that this part is ready
            if (threadIdx.x < nsplit && threadIdx.x != split) mbar_arrive_remote(dsmem_addr(bar(kParts), threadIdx.x));
            if (grp == 0) {
                // group 0 merges heads h = split + j nk (j < nh) of every part:
                // w_s = 2^(m_s - M) over the non-empty parts, out = sum_s w_s O_s / sum_s w_s l_s
                const int nh = (NH - split + nk - 1) / nk;
                const bool pok = warp_wait_cluster(bar(kParts), 0u, p.wait_ns, abort_flag, p.flags);
                float* const wts = reinterpret_cast<float*>(smem + (q_s - bar0));  // [kMcMaxCluster + 1][NH]
                if (wq == 0 && pok && lane < nh) {
                    const int h = split + lane * nk;
                    float ms[kMcMaxCluster], ls[kMcMaxCluster];
#pragma unroll
                    for (int s = 0; s < kMcMaxCluster; ++s) {
                        ms[s] = -INFINITY;
                        ls[s] = 0.f;
                        if (s < nk) {
                            const float* q = dsmem_ptr(part_p + NH * D + 2 * h, static_cast<uint32_t>(s));
                            ms[s] = q[0];
                            ls[s] = q[1];
                        }
                    }
                    float M = -INFINITY;
#pragma unroll
                    for (int s = 0; s < kMcMaxCluster; ++s)
                        if (ls[s] > 0.f) M = fmaxf(M, ms[s]);
                    float den = 0.f;
#pragma unroll
                    for (int s = 0; s < kMcMaxCluster; ++s) {
                        const float w = ls[s] > 0.f ? exp2f(ms[s] - M) : 0.f;
                        wts[s * NH + lane] = w;
                        den += w * ls[s];
                    }
                    wts[kMcMaxCluster * NH + lane] = den > 0.f ? 1.f / den : 0.f;
                }
                if (!bar_any(gbar, 128, !pok || any_gave_up)) {
                    constexpr int kMaxH = NH / 2;  // heads per split when nk = 2
                    float acc[kMaxH];
#pragma unroll
                    for (int jj = 0; jj < kMaxH; ++jj) acc[jj] = 0.f;
#pragma unroll
                    for (int s = 0; s < kMcMaxCluster; ++s) {
                        if (s < nk) {  // the loads of all parts can be in flight together
                            const float* src = dsmem_ptr(part_p + dd, static_cast<uint32_t>(s));
                            float v[kMaxH];
#pragma unroll
                            for (int jj = 0; jj < kMaxH; ++jj) v[jj] = jj < nh ? src[(split + jj * nk) * D] : 0.f;
#pragma unroll
                            for (int jj = 0; jj < kMaxH; ++jj) acc[jj] += wts[s * NH + jj] * v[jj];
                        }
                    }
#pragma unroll
                    for (int jj = 0; jj < kMaxH; ++jj) {
                        const int h = split + jj * nk;
                        if (jj < nh && h < gh)
                            p.out[b * p.out_sb + static_cast<int64_t>(qh0 + h) * p.out_sh + dd] =
                                __float2bfloat16_rn(acc[jj] * wts[kMcMaxCluster * NH + jj]);
                    }
                }
            }
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
    if (p.cluster) {
        if (!cluster_waited) cluster_wait();  // phase 0, for the warps that did not merge
        // phase 1: no CTA of the cluster leaves while split 0 may still read its part
        cluster_arrive();
        cluster_wait();
    }
}

}  // namespace apd
