// apd_api.cu -- the C ABI of libattn_paged_decode.so: argument validation,
// launch planning, TMA descriptor encoding and the two kernel launches.
//
// The entry point and its checks follow the AstrAI commit log of
// csrc/kernels/attn_paged_decode.cu: a thin binding that validates
// q_head % kv_head == 0 and head-dim contiguity, checks the split-KV scratch
// and output layout, runs on the caller's stream, and never allocates inside a
// decode step (the partials live in a preallocated workspace, which is what lets
// the decode step be captured in a CUDA graph).
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <cmath>
#include <cstddef>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "../../include/attn_paged_decode.h"
#include "apd_decode_tc.cuh"
#include "apd_gemv.cuh"
#include "apd_kernels.cuh"
#include "apd_prefill_tc.cuh"
#include "apd_prefill.cuh"

namespace {

thread_local char g_last_cuda_error[512] = "";

int cuda_fail(cudaError_t e, const char* what) {
    std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s: %s", what, cudaGetErrorString(e));
    return APD_ERR_CUDA;
}

int driver_fail(int code, const char* what) {
    std::snprintf(g_last_cuda_error, sizeof g_last_cuda_error, "%s: CUresult %d", what, code);
    return APD_ERR_CUDA;
}

constexpr size_t kSmemLimit = 232448;  // sm_100a: 227 KB of opt-in shared memory per block
constexpr size_t kWsAlign = 256;
constexpr int kDefaultSmCount = 148;   // B200

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct Traits {
    int stages;
    int max_warps;
};

// One ring per warp.  D = 32 and 64 are latency-bound per warp, so more warps beat deeper
// rings (B200, 268 MB of K/V, graph-timed): D = 32, g = 4: 8 warps x 4 stages 55.3 us,
// 12 x 3 52.9 us; g = 32: 62.8 -> 52.4 us.  D = 64, g = 4: 8 x 4 (6 fit) 50.4 us, 10 x 2
// 48.7 us; g = 1: 50.0 -> 46.1 us.  The kernels are instantiated with these stages, so
// this table is their single source.
constexpr Traits traits_for(int D) {
    return D == 32 ? Traits{3, 12} : D == 64 ? Traits{2, 10} : D == 128 ? Traits{3, 6} : Traits{2, 4};
}

// The shared-ring layout (balanced mode, g > 16): K/V stages per kv head and the most
// warps per CTA; {0, 0} = not used for this head dim.  Measured on B200 (B = 16,
// 268 MB of K/V, graph-timed): these warps per SM are latency-bound, so more warps beat
// deeper rings.  D = 128, g = 32: 8 warps x 2 stages 64.3 us, 6 x 3 75.3 us, 4 x 3 or 4 x 4
// 84-85 us, one ring per warp 97.8 us.  D = 32 keeps one ring per warp (71.6 us against
// 77.1 shared): its short tiles leave a warp pair with too little work per wait.
constexpr Traits share_traits_for(int D) {
    return D == 32 ? Traits{0, 0} : D == 64 ? Traits{4, 8} : D == 128 ? Traits{2, 8} : Traits{2, 4};
}
template <int D>
constexpr int kStages = traits_for(D).stages;

// The unit kernel (one CTA per unit, or per split with fixed splits) at D = 32 takes 16 warps
// x 2 stages: B = 16 at 268 MB of K/V, one CTA per unit, 46.7 -> 44.0 us against 12 x 3 (14 x 3
// 46.1, 11 x 4 49.5).  The balanced split kernel keeps 12 x 3 (16 x 2 took 50.9 -> 52.0 us).
constexpr Traits unit_traits_for(int D) { return D == 32 ? Traits{2, 16} : traits_for(D); }
template <int D>
constexpr int kUnitStages = unit_traits_for(D).stages;
template <int D>
constexpr int kShareStages = share_traits_for(D).stages;

// A plan never asks for more warps than the kernel's launch bound allows.
static_assert(traits_for(32).max_warps <= apd::kMaxWarpsD<32, false> &&
                  traits_for(64).max_warps <= apd::kMaxWarpsD<64, false> &&
                  traits_for(128).max_warps <= apd::kMaxWarpsD<128, false> &&
                  traits_for(256).max_warps <= apd::kMaxWarpsD<256, false>,
              "warps per CTA above the split kernel's launch bound");
static_assert(unit_traits_for(32).max_warps <= apd::kMaxWarpsD<32, false>,
              "warps per CTA above the unit kernel's launch bound");
static_assert(share_traits_for(64).max_warps <= apd::kMaxWarpsD<64, true> &&
                  share_traits_for(128).max_warps <= apd::kMaxWarpsD<128, true> &&
                  share_traits_for(256).max_warps <= apd::kMaxWarpsD<256, true>,
              "warps per CTA above the shared-ring kernel's launch bound");

bool head_dim_ok(int D) { return D == 32 || D == 64 || D == 128 || D == 256; }

// the binding mirrors apd_plan field by field
static_assert(sizeof(apd_plan) == 72 && offsetof(apd_plan, q_heads_per_block) == 68, "apd_plan layout");

struct Shape {
    int B, Hq, Hkv, D, g, HB, rows_max;
    int64_t units;  // B * Hkv * HB
};

int make_shape(int B, int Hq, int Hkv, int D, Shape* s) {
    if (B < 0 || Hq <= 0 || Hkv <= 0) return APD_ERR_SHAPE;
    if (Hq % Hkv != 0) return APD_ERR_GQA;
    if (!head_dim_ok(D)) return APD_ERR_HEAD_DIM;
    if (B > APD_MAX_BATCH) return APD_ERR_TOO_LARGE;
    s->B = B;
    s->Hq = Hq;
    s->Hkv = Hkv;
    s->D = D;
    s->g = Hq / Hkv;
    s->HB = (s->g + apd::kMaxRows - 1) / apd::kMaxRows;
    s->rows_max = s->g < apd::kMaxRows ? s->g : apd::kMaxRows;
    s->units = static_cast<int64_t>(B) * Hkv * s->HB;
    return APD_OK;
}

uint32_t q_tile_bytes(const Shape& s) { return static_cast<uint32_t>(align_up(static_cast<size_t>(s.rows_max) * s.D * 2, 1024)); }
uint32_t stage_bytes(const Shape& s) { return 2u * apd::kTile * s.D * 2u + q_tile_bytes(s); }

// share: the layout where the HB warps of a kv head share one K/V ring (the balanced mode
// when g > 16): warps / HB K/V rings and `warps` Q rings, and an `empty` mbarrier per stage.
size_t smem_bytes(const Shape& s, int warps, int stages, bool share = false) {
    // mbarriers (full, and empty in the shared layout), the abort word (8 bytes), lengths and
    // prefix sums
    const size_t meta = 8ull * warps * stages * (share ? 2 : 1) + 8 + 4ull * (2ull * s.B + 1);
    const size_t rings = share ? static_cast<size_t>(warps / s.HB) * stages * (2ull * apd::kTile * s.D * 2) +
                                     static_cast<size_t>(warps) * stages * q_tile_bytes(s)
                               : static_cast<size_t>(warps) * stages * stage_bytes(s);
    return align_up(meta, 16) + 1024 + rings;
}

// The one-CTA-per-unit kernel (unit_kernel): full mbarriers, the merge mbarrier, the abort
// word and tile counter (8 bytes), the claimed tile of each stage, then the per-warp rings.
size_t unit_smem_bytes(const Shape& s, int warps, int stages) {
    const size_t meta = 8ull * warps * stages + 8 + 8 + 4ull * warps * stages;
    return align_up(meta, 16) + 1024 + static_cast<size_t>(warps) * stages * stage_bytes(s);
}

// The most warps per CTA that fit (a multiple of HB in the shared layout), or 0.
int warps_for(const Shape& s, bool share = false) {
    const Traits t = share ? share_traits_for(s.D) : traits_for(s.D);
    if (t.stages < 1) return 0;
    for (int w = t.max_warps; w >= 1; --w)
        if ((!share || w % s.HB == 0) && smem_bytes(s, w, t.stages, share) <= kSmemLimit) return w;
    return 0;
}

// Workspace: [flags header 256 B][cum (B+1) int32][o_part][ml_part], each 256-aligned.
size_t ws_head_bytes(const Shape& s) { return kWsAlign + align_up(4ull * (s.B + 1), kWsAlign); }
size_t ws_bytes_for(const Shape& s, int64_t slots) {
    return ws_head_bytes(s) + align_up(static_cast<size_t>(slots) * s.rows_max * s.D * 4, kWsAlign) +
           align_up(static_cast<size_t>(slots) * s.rows_max * 2 * 4, kWsAlign);
}
int64_t slots_fitting(const Shape& s, size_t bytes) {
    if (bytes < ws_head_bytes(s)) return -1;
    const size_t per = static_cast<size_t>(s.rows_max) * (s.D + 2) * 4;
    int64_t n = static_cast<int64_t>((bytes - ws_head_bytes(s)) / per);
    while (n > 0 && ws_bytes_for(s, n) > bytes) --n;
    return n;
}

struct Plan {
    int mode, ksplit, workers, groups, ctas, warps, stages, combine_ctas;
    int cluster = 0;  // mode 3: CTAs per cluster (the splits of a unit, merged over DSMEM), or 0
    int hblocks = 1;  // mode 3: q-head blocks per kv head (CTAs per split of a (sequence, kv head))
    int hb_heads = 0; // mode 3: q heads per block (a multiple of 16, at most 64)
    bool share;  // balanced mode, g > 16: a kv head's HB warps share one K/V ring
    size_t smem;
    int64_t slots;
    size_t ws_needed;
};

// One-CTA-per-unit plan (mode 2, unit_kernel): CTA u owns unit u, its warps claim the
// unit's tiles from a shared counter and merge their parts in shared memory; a single
// launch, no partials in the workspace.
// The unit kernel's geometry: the most warps (up to the head dim's maximum) whose rings fit.
void unit_geometry(const Shape& s, Plan* pl) {
    pl->share = false;
    pl->stages = unit_traits_for(s.D).stages;
    pl->warps = unit_traits_for(s.D).max_warps;
    while (pl->warps > 1 && unit_smem_bytes(s, pl->warps, pl->stages) > kSmemLimit) --pl->warps;
    pl->smem = unit_smem_bytes(s, pl->warps, pl->stages);
}

void cta_local_plan(const Shape& s, Plan* pl) {
    pl->mode = 2;
    unit_geometry(s, pl);
    pl->ksplit = pl->warps;
    pl->groups = 0;
    pl->workers = static_cast<int>(s.units * pl->warps);
    pl->ctas = static_cast<int>(s.units);
    pl->slots = 0;
    pl->combine_ctas = 0;
}

// Whether the one-CTA-per-unit plan beats the balanced plan `pl` for these host-known lengths
// (clamped to [0, len_cap] as the kernels clamp them).  Only when every unit gets a CTA of
// its own on a distinct SM, a kv head has one head block (with more, each block's CTA would
// stream the kv head's K/V again: g = 32 measured 187 against 62 us), and the longest unit
// is at most the share per CTA of a launch on max(units, 7/8 of the SMs) CTAs (so that a
// few long units, which would leave most SMs idle, do not qualify) plus about what the
// combine kernel costs: 3% and 1024 / D tiles.  Measured on B200 at 268 MB of K/V, 128
// equal units: D = 32 53.4 -> 49.7 us, D = 64 48.5 -> 43.9 us, D = 128 46.2 -> 43.9 us,
// D = 256 49.2 -> 45.7 us against the balanced plan.
bool cta_local_wins(const Shape& s, const Plan& pl, int sm_count, const int32_t* host_lens, int64_t len_cap) {
    if (s.units > sm_count || pl.ctas < 1 || s.HB > 1) return false;
    // a part's (m, l) and accumulator rows go to its warp's ring once the stream ends
    if (128ull + 4ull * s.rows_max * (s.D + 8) > static_cast<size_t>(unit_traits_for(s.D).stages) * stage_bytes(s))
        return false;
    const int64_t ups = static_cast<int64_t>(s.Hkv) * s.HB;
    int64_t total = 0, longest = 0;
    for (int b = 0; b < s.B; ++b) {
        const int64_t L = std::min<int64_t>(std::max<int32_t>(host_lens[b], 0), len_cap);
        const int64_t n = (L + apd::kTile - 1) / apd::kTile;
        total += n * ups;
        longest = std::max(longest, n);
    }
    const int64_t ctas = std::max<int64_t>(s.units, static_cast<int64_t>(sm_count) * 7 / 8);
    const int64_t share = (total + ctas - 1) / ctas;
    return 32 * longest <= 33 * share + 32 * (1024 / s.D);
}

// Tensor-core multi-query plan (mode 3, decode_mq_tc_kernel): kv heads with more than 16
// query heads at D = 128.  One CTA per split of each (sequence, kv head, q-head block); its
// 128-token tiles meet all the block's query heads (padded to NH = 32 or 64) in one tcgen05
// MMA, where the split kernel needs a head block of 16 per warp.  Up to 64 query heads are
// one block; above that, ceil(g / 64) blocks of ceil(g / blocks) heads rounded up to 16, so
// that every block starts on a 16-row boundary of the partial slots.  The partials take the
// fixed-split slots (the 16-row head blocks' rows of each split), so the combine is the
// fixed-split one.
template <int NH>
using McShapeT = apd::McShape<128, NH>;

constexpr int kMcBlockHeads = 64;  // most q heads of one tensor-core decode CTA
int mq_tc_hblocks(const Shape& s) { return (s.g + kMcBlockHeads - 1) / kMcBlockHeads; }
int mq_tc_block_heads(const Shape& s) {
    const int nb = mq_tc_hblocks(s);
    return ((s.g + nb - 1) / nb + apd::kMaxRows - 1) / apd::kMaxRows * apd::kMaxRows;
}
// NH of the tensor-core kernel for this shape, or 0 when the shape does not take it
int mq_tc_heads(const Shape& s) {
    return s.D == 128 && s.g > 16 ? (mq_tc_block_heads(s) <= 32 ? 32 : 64) : 0;
}
bool mq_tc_eligible(const Shape& s) { return mq_tc_heads(s) > 0; }
// Co-resident clusters of k tensor-core decode CTAs, per NH (index 0: 32 heads, 1: 64).
struct McCaps {
    int c[2][apd::kMcMaxCluster + 1];
};

// Splits per unit with automatic splitting: the (sequence, kv head, q-head block) units
// spread over 7/8 of the SMs (the rate at which D = 128 streams best, as in the balanced
// plan), at most one split per 128-token tile the page table can address, and no more than
// the workspace holds.  Returns 0 when the workspace holds no partials at all and the unit
// count needs some.
int64_t mq_tc_auto_splits(const Shape& s, int sm_count, size_t ws_bytes, int64_t tiles_bound) {
    const int64_t u2 = static_cast<int64_t>(s.B) * s.Hkv * mq_tc_hblocks(s);
    int64_t k = std::max<int64_t>(1, static_cast<int64_t>(sm_count) * 7 / 8 / std::max<int64_t>(1, u2));
    if (tiles_bound >= 0) {
        const int64_t per_unit = tiles_bound / std::max<int64_t>(1, s.units);  // 32-token tiles
        k = std::min<int64_t>(k, std::max<int64_t>(1, (per_unit + 3) / 4));
    }
    if (ws_bytes != SIZE_MAX && k > 1) {
        const int64_t fit = slots_fitting(s, ws_bytes) / std::max<int64_t>(1, s.units);
        k = std::max<int64_t>(1, std::min(k, fit));
    }
    return k;
}

void mq_tc_plan(const Shape& s, int64_t ksplit, int sm_count, int cluster, Plan* pl);

// Whether the splits of every unit can be one cluster of `k` CTAs that the device runs all
// at once (cluster_caps[k]: clusters of k of the kernel's CTAs that fit the device at the
// same time; without it, every k SMs are assumed to hold one).  Then the splits merge over
// DSMEM in the kernel: measured on B200 (gqa32), the separate combine kernel costs 4.5 of
// 49.6 us per call.
int mq_tc_cluster(const Shape& s, int64_t k, int sm_count, const McCaps* caps) {
    if (k < 2 || k > apd::kMcMaxCluster) return 0;
    const int64_t cap = caps ? caps->c[mq_tc_heads(s) == 64 ? 1 : 0][k] : sm_count / k;
    return static_cast<int64_t>(s.B) * s.Hkv * mq_tc_hblocks(s) <= cap ? static_cast<int>(k) : 0;
}

// Warps of a combine CTA: enough for one batch of kCombineBatch partial slots per warp,
// 4 to 16.  A unit has about groups / B partials in the balanced mode (each sequence's
// share of the groups, plus the one it starts in) and num_splits in the fixed mode.
// Measured (llama8b-shaped, L = 4096, graph-timed): 8 warps at 4 partials per unit cost
// llama8b 45.9 -> 48.2 us and ragged 332 -> 345-353 us, so 4 stays the floor.
int64_t partials_per_unit(const Shape& s, const Plan& pl) {
    return pl.mode == 0 ? pl.groups / std::max(1, s.B) + 1 : pl.ksplit;
}
int combine_warps(const Shape& s, const Plan& pl) {
    const int64_t per_unit = partials_per_unit(s, pl);
    int w = 4;
    while (w < 16 && static_cast<int64_t>(w) * apd::kCombineBatch < per_unit) w *= 2;
    return w;
}

// With at most one batch of partials per unit, a grid of a few CTAs per SM that walk the
// units (each warp merging whole rows) beats one CTA per (unit, row): the large-batch plans
// have about one partial per unit, and most of their units are covered by one warp, so most
// row CTAs would only return.  Graph-timed on B200: ragged (B = 128, 64/8 heads) 414-419 ->
// 409-410 us per call; the llama8b-shaped batch without host lengths (5 partials per unit)
// went 46.0 -> 46.6 us, so it keeps one CTA per (unit, row).
bool combine_per_unit(const Shape& s, const Plan& pl) {
    return partials_per_unit(s, pl) <= apd::kCombineBatch;
}
constexpr int kCombineUnitCtasPerSm = 4;
int64_t combine_unit_ctas(const Shape& s, int sm_count) {
    return std::min<int64_t>(s.units, static_cast<int64_t>(sm_count) * kCombineUnitCtasPerSm);
}

void mq_tc_plan(const Shape& s, int64_t ksplit, int sm_count, int cluster, Plan* pl) {
    pl->mode = 3;
    pl->cluster = cluster;
    pl->share = false;
    pl->ksplit = static_cast<int>(ksplit);
    pl->groups = 0;
    const bool h64 = mq_tc_heads(s) == 64;
    pl->warps = (h64 ? McShapeT<64>::kThreads : McShapeT<32>::kThreads) / 32;
    pl->stages = h64 ? McShapeT<64>::kVStages : McShapeT<32>::kVStages;
    pl->smem = h64 ? McShapeT<64>::kSmemBytes : McShapeT<32>::kSmemBytes;
    pl->hblocks = mq_tc_hblocks(s);
    pl->hb_heads = mq_tc_block_heads(s);
    pl->ctas = static_cast<int>(static_cast<int64_t>(s.B) * s.Hkv * pl->hblocks * ksplit);
    pl->workers = pl->ctas;
    // the partial slots are reserved whether or not the merge runs over DSMEM, so that the
    // workspace a split count needs does not depend on the device's cluster placement
    pl->slots = ksplit >= 2 ? s.units * ksplit : 0;
    pl->combine_ctas = ksplit >= 2 && cluster == 0
                           ? static_cast<int>(combine_per_unit(s, *pl) ? combine_unit_ctas(s, sm_count)
                                                                      : s.units * s.rows_max)
                           : 0;
}

// tiles_bound: an upper bound on the number of tiles (host-known), or -1.
// host_lens: NULL, or the B sequence lengths as the host knows them (a planning hint;
// the kernels read the device lengths), clamped to len_cap.
// allow_tc: the tensor-core multi-query plan may be chosen (the shared-ring self-test turns
// it off to reach the shared ring).
int make_plan(const Shape& s, int num_splits, int sm_count, size_t ws_bytes, int64_t tiles_bound, Plan* pl,
              const int32_t* host_lens = nullptr, int64_t len_cap = 0, bool allow_tc = true,
              const McCaps* cluster_caps = nullptr) {
    if (num_splits < 0) return APD_ERR_NUM_SPLITS;
    if (allow_tc && mq_tc_eligible(s)) {
        const int64_t k = num_splits > 0 ? num_splits : mq_tc_auto_splits(s, sm_count, ws_bytes, tiles_bound);
        if (static_cast<int64_t>(s.B) * s.Hkv * mq_tc_hblocks(s) * k > INT32_MAX / 64) return APD_ERR_TOO_LARGE;
        mq_tc_plan(s, k, sm_count, mq_tc_cluster(s, k, sm_count, cluster_caps), pl);
        pl->ws_needed = ws_bytes_for(s, pl->slots);
        if (ws_bytes != SIZE_MAX && ws_bytes < pl->ws_needed) return APD_ERR_WORKSPACE;
        return APD_OK;
    }
    const Traits t = traits_for(s.D);
    pl->stages = t.stages;
    pl->warps = warps_for(s);
    if (pl->warps < 1) return APD_ERR_TOO_LARGE;
    pl->smem = smem_bytes(s, pl->warps, pl->stages);
    pl->share = false;
    if (num_splits == 0) {
        // Balanced mode: groups of Hkv * HB warps (one per kv head and head block)
        // share the sequence-tile positions equally; as many groups as fit the
        // device's resident warps, the known tile bound and the workspace.
        pl->mode = 0;
        pl->ksplit = 0;
        if (s.HB > 1 && warps_for(s, true) > 0) {
            // the HB warps of a kv head walk the same positions: one K/V stream for them
            pl->share = true;
            pl->stages = share_traits_for(s.D).stages;
            pl->warps = warps_for(s, true);
            pl->smem = smem_bytes(s, pl->warps, pl->stages, true);
        }
        const int64_t ups = static_cast<int64_t>(s.Hkv) * s.HB;
        // D = 128 streams HBM with spare per-SM issue capacity: it runs fastest on
        // 7/8 of the SMs (measured on B200: 128 of 148 CTAs is 5-9% faster than 148
        // for the llama8b, long-context and large-batch shapes, because with every SM
        // streaming some SMs get a systematically smaller share of the bandwidth and
        // the equal static split waits for them).  D = 32/64/256 are bound by per-tile
        // latency and want every SM.
        const int64_t resident = static_cast<int64_t>(sm_count) * pl->warps;
        const int64_t budget = (s.D == 128) ? resident * 7 / 8 : resident;
        int64_t groups = std::max<int64_t>(1, budget / ups);
        if (tiles_bound >= 0) groups = std::min<int64_t>(groups, std::max<int64_t>(1, tiles_bound / ups));
        if (ws_bytes != SIZE_MAX) {
            const int64_t cap = slots_fitting(s, ws_bytes) / (2 * ups);
            if (cap < 1) return APD_ERR_WORKSPACE;
            groups = std::min(groups, cap);
        }
        if (groups * ups > INT32_MAX / 4) return APD_ERR_TOO_LARGE;
        pl->groups = static_cast<int>(groups);
        const int64_t workers = groups * ups;
        pl->workers = static_cast<int>(workers);
        pl->slots = 2 * workers;
        // one group covers every position: no unit is split, every warp writes its
        // output directly, and the call is a single launch (the unsplit path)
        pl->combine_ctas = groups > 1 ? static_cast<int>(combine_per_unit(s, *pl) ? combine_unit_ctas(s, sm_count)
                                                                                 : s.units * s.rows_max)
                                      : 0;
        pl->ctas = (pl->workers + pl->warps - 1) / pl->warps;
        if (host_lens && pl->combine_ctas > 0 && cta_local_wins(s, *pl, sm_count, host_lens, len_cap))
            cta_local_plan(s, pl);
    } else {
        // fixed splits: one unit-kernel CTA per split of each unit
        pl->mode = 1;
        pl->ksplit = num_splits;
        pl->groups = 0;
        unit_geometry(s, pl);
        const int64_t ctas = s.units * num_splits;
        if (ctas > INT32_MAX / 64) return APD_ERR_TOO_LARGE;
        pl->ctas = static_cast<int>(ctas);
        pl->workers = static_cast<int>(ctas * pl->warps);
        pl->slots = num_splits >= 2 ? ctas : 0;
        pl->combine_ctas = num_splits >= 2 ? static_cast<int>(combine_per_unit(s, *pl) ? combine_unit_ctas(s, sm_count)
                                                                                        : s.units * s.rows_max)
                                           : 0;
    }
    if (pl->mode == 0) pl->ctas = (pl->workers + pl->warps - 1) / pl->warps;
    pl->ws_needed = ws_bytes_for(s, pl->slots);
    if (ws_bytes != SIZE_MAX && ws_bytes < pl->ws_needed) return APD_ERR_WORKSPACE;
    return APD_OK;
}

// ---------------------------------------------------------------- devices
struct DeviceState {
    bool init = false;
    int sm_count = 0;
    bool smem_attr_set[16] = {};  // head dim x {split kernel, with shared rings, unit kernel, unit kernel with fixed splits}
    bool mq_tc_attr_set[2] = {false, false};  // NH = 32, 64
    bool mq_caps_init = false;
    McCaps mq_caps = {};  // co-resident clusters of k tensor-core decode CTAs
    bool gemv_attr_set = false;
    bool prefill_attr_set[4] = {false, false, false, false};
    bool prefill_tc_attr_set[4] = {false, false, false, false};
    bool prefill_tc2_attr_set[4] = {false, false, false, false};
};
std::mutex g_mu;
DeviceState g_devices[128];

int device_state(DeviceState** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 128) return APD_ERR_ARGUMENT;
    std::lock_guard<std::mutex> lock(g_mu);
    DeviceState& d = g_devices[dev];
    if (!d.init) {
        e = cudaDeviceGetAttribute(&d.sm_count, cudaDevAttrMultiProcessorCount, dev);
        if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute(MultiProcessorCount)");
        d.init = true;
    }
    *out = &d;
    return APD_OK;
}

// Clusters of k tensor-core decode CTAs that the device runs at the same time, k = 2..8
// (cudaOccupancyMaxActiveClusters; 0 where the query fails).  Computed once per device.
template <int NH>
void mq_query_caps(DeviceState* d, int* caps) {
    auto kern = apd::decode_mq_tc_kernel<128, NH>;
    const int hi = NH == 64 ? 1 : 0;
    if (!d->mq_tc_attr_set[hi]) {
        if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 static_cast<int>(McShapeT<NH>::kSmemBytes)) == cudaSuccess)
            d->mq_tc_attr_set[hi] = true;
    }
    for (int c = 2; c <= apd::kMcMaxCluster; ++c) {
        cudaLaunchAttribute attr;
        attr.id = cudaLaunchAttributeClusterDimension;
        attr.val.clusterDim.x = static_cast<unsigned>(c);
        attr.val.clusterDim.y = 1;
        attr.val.clusterDim.z = 1;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(c * d->sm_count));
        cfg.blockDim = dim3(static_cast<unsigned>(McShapeT<NH>::kThreads));
        cfg.dynamicSmemBytes = McShapeT<NH>::kSmemBytes;
        cfg.attrs = &attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (!d->mq_tc_attr_set[hi] || cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess) n = 0;
        caps[c] = n;
    }
}
const McCaps* mq_cluster_caps(DeviceState* d) {
    std::lock_guard<std::mutex> lock(g_mu);
    if (!d->mq_caps_init) {
        mq_query_caps<32>(d, d->mq_caps.c[0]);
        mq_query_caps<64>(d, d->mq_caps.c[1]);
        cudaGetLastError();  // a failed query only turns the cluster merge off
        d->mq_caps_init = true;
    }
    return &d->mq_caps;
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &ptr, 12000, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    });
    return fn;
}

// ---------------------------------------------------------------- validation
bool is_null(const apd_tensor* t) { return t == nullptr || t->data == nullptr; }

// Strides with extent-1 dimensions replaced by the contiguous value, so that
// any stride a framework reports for a broadcast / size-1 dim is accepted.
void normalized_strides(const apd_tensor* t, int64_t* st) {
    int64_t inner = 1;
    for (int i = t->ndim - 1; i >= 0; --i) {
        st[i] = (t->shape[i] == 1) ? inner : t->stride[i];
        inner *= t->shape[i];
    }
}

// Head dim contiguous, every other stride positive and a multiple of 8
// elements (16 bytes), base 16-byte aligned.
bool aligned_bf16_layout(const apd_tensor* t, int64_t* st) {
    normalized_strides(t, st);
    if (st[t->ndim - 1] != 1) return false;
    for (int i = 0; i < t->ndim - 1; ++i)
        if (st[i] <= 0 || st[i] % 8 != 0 || st[i] * 2 >= (1ll << 40)) return false;
    return (reinterpret_cast<uintptr_t>(t->data) & 15u) == 0;
}

struct Validated {
    Shape s;
    int P, NP, MP;
    int64_t qst[3], kst[4], vst[4], ost[3], pst[2];
};

// Checks the call's descriptors.  pt == nullptr selects the contiguous-KV form:
// k/v are [B, Lmax, Hkv, D] (one "page" of Lmax tokens per sequence, page b for
// sequence b), and Lmax need not be a multiple of 32.
int validate(const apd_tensor* q, const apd_tensor* k, const apd_tensor* v, const apd_tensor* pt,
             const apd_tensor* sl, const apd_tensor* out, int num_splits, Validated* V) {
    const bool contig = (pt == nullptr);
    if (!q || !k || !v || !sl || !out) return APD_ERR_NULL_POINTER;
    const bool empty_batch = (q->ndim >= 1 && q->shape[0] == 0);
    if ((is_null(k) || is_null(v)) && !(contig && empty_batch)) return APD_ERR_NULL_POINTER;
    // The per-sequence tensors may be empty (and NULL) only when the batch is empty.
    if ((is_null(q) || (!contig && is_null(pt)) || is_null(sl) || is_null(out)) && !empty_batch)
        return APD_ERR_NULL_POINTER;
    if (q->dtype != APD_DTYPE_BF16 || k->dtype != APD_DTYPE_BF16 || v->dtype != APD_DTYPE_BF16 ||
        out->dtype != APD_DTYPE_BF16 || (!contig && pt->dtype != APD_DTYPE_INT32) || sl->dtype != APD_DTYPE_INT32)
        return APD_ERR_DTYPE;
    if (q->ndim != 3 || out->ndim != 3 || k->ndim != 4 || v->ndim != 4 || (!contig && pt->ndim != 2) ||
        sl->ndim != 1)
        return APD_ERR_SHAPE;
    for (int i = 0; i < 3; ++i)
        if (q->shape[i] != out->shape[i] || q->shape[i] < 0) return APD_ERR_SHAPE;
    const int64_t B = q->shape[0], Hq = q->shape[1], D = q->shape[2];
    for (int i = 0; i < 4; ++i)
        if (k->shape[i] != v->shape[i] || (k->shape[i] <= 0 && !(contig && i == 0 && B == 0))) return APD_ERR_SHAPE;
    const int64_t NP = k->shape[0], P = k->shape[1], Hkv = k->shape[2];
    const int64_t MP = contig ? 1 : pt->shape[1];
    if (k->shape[3] != D || sl->shape[0] != B) return APD_ERR_SHAPE;
    if (contig ? (NP != B) : (pt->shape[0] != B || MP <= 0)) return APD_ERR_SHAPE;
    if (Hq <= 0 || D <= 0) return APD_ERR_SHAPE;
    if (Hq > INT32_MAX || Hkv > INT32_MAX || NP > INT32_MAX || P > INT32_MAX || MP > INT32_MAX)
        return APD_ERR_TOO_LARGE;
    if (B > APD_MAX_BATCH) return APD_ERR_TOO_LARGE;
    int rc = make_shape(static_cast<int>(B), static_cast<int>(Hq), static_cast<int>(Hkv), static_cast<int>(D), &V->s);
    if (rc) return rc;
    // A 32-token tile must not straddle two pages (one page-table lookup per tile).
    if (!contig && P % apd::kTile != 0) return APD_ERR_PAGE_SIZE;
    if (num_splits < 0) return APD_ERR_NUM_SPLITS;
    if (!aligned_bf16_layout(q, V->qst) || !aligned_bf16_layout(out, V->ost) || !aligned_bf16_layout(k, V->kst) ||
        !aligned_bf16_layout(v, V->vst))
        return APD_ERR_LAYOUT;
    if (contig) {
        V->pst[0] = V->pst[1] = 0;
    } else {
        normalized_strides(pt, V->pst);
        if (V->pst[0] < 0 || V->pst[1] < 0 || (reinterpret_cast<uintptr_t>(pt->data) & 3u)) return APD_ERR_LAYOUT;
    }
    int64_t sst[1];
    normalized_strides(sl, sst);
    if (sst[0] != 1 || (reinterpret_cast<uintptr_t>(sl->data) & 3u)) return APD_ERR_LAYOUT;
    // flattened tile indices must fit in int32 on the device
    const int64_t tiles_bound = V->s.units * MP * ((P + apd::kTile - 1) / apd::kTile);
    if (tiles_bound >= INT32_MAX / 2) return APD_ERR_TOO_LARGE;
    V->P = static_cast<int>(P);
    V->NP = static_cast<int>(NP);
    V->MP = static_cast<int>(MP);
    return APD_OK;
}

// ---------------------------------------------------------------- TMA maps
// K/V: D >= 64 -> 5-D view {64, Hkv, P, NP, D/64}, box {64, 1, 32, 1, D/64},
//      128-byte swizzle: one box = one [32 x D] tile of one kv head, landing in
//      shared memory as D/64 blocks of [32 tokens][64 elements].
//      D == 32 -> 4-D view {32, Hkv, P, NP}, box {32, 1, 32, 1}, 64-byte swizzle.
// box_blocks < D/64 (D >= 64): a box holds that many 64-dim blocks instead (the
// tensor-core prefill loads one block per box so the tile's rows of one block are
// contiguous).
int encode_kv_map(CUtensorMap* map, const apd_tensor* t, const int64_t* st, int D, int box_blocks = 0) {
    auto fn = encode_fn();
    if (!fn) return driver_fail(-1, "cuTensorMapEncodeTiled entry point");
    cuuint64_t dims[5], strides[4];
    cuuint32_t box[5], estr[5] = {1, 1, 1, 1, 1};
    cuuint32_t rank;
    CUtensorMapSwizzle swz;
    if (D >= 64) {
        rank = 5;
        dims[0] = 64; dims[1] = t->shape[2]; dims[2] = t->shape[1]; dims[3] = t->shape[0]; dims[4] = D / 64;
        strides[0] = st[2] * 2; strides[1] = st[1] * 2; strides[2] = st[0] * 2; strides[3] = 128;
        box[0] = 64; box[1] = 1; box[2] = apd::kTile; box[3] = 1; box[4] = box_blocks > 0 ? box_blocks : D / 64;
        swz = CU_TENSOR_MAP_SWIZZLE_128B;
    } else {
        rank = 4;
        dims[0] = 32; dims[1] = t->shape[2]; dims[2] = t->shape[1]; dims[3] = t->shape[0];
        strides[0] = st[2] * 2; strides[1] = st[1] * 2; strides[2] = st[0] * 2;
        box[0] = 32; box[1] = 1; box[2] = apd::kTile; box[3] = 1;
        swz = CU_TENSOR_MAP_SWIZZLE_64B;
    }
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, t->data, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return driver_fail(r, "cuTensorMapEncodeTiled(kv)");
    return APD_OK;
}

// Q: D >= 64 -> 4-D view {64, Hq, B, D/64}, box {64, rows_max, 1, D/64}
//    (D/64 blocks of [rows_max][64] in shared memory);
//    D == 32 -> 3-D view {32, Hq, B}, box {32, rows_max, 1}.
int encode_q_map(CUtensorMap* map, const apd_tensor* t, const int64_t* st, int D, int rows_max) {
    auto fn = encode_fn();
    if (!fn) return driver_fail(-1, "cuTensorMapEncodeTiled entry point");
    cuuint64_t dims[4], strides[3];
    cuuint32_t box[4], estr[4] = {1, 1, 1, 1};
    cuuint32_t rank;
    CUtensorMapSwizzle swz;
    if (D >= 64) {
        rank = 4;
        dims[0] = 64; dims[1] = t->shape[1]; dims[2] = t->shape[0]; dims[3] = D / 64;
        strides[0] = st[1] * 2; strides[1] = st[0] * 2; strides[2] = 128;
        box[0] = 64; box[1] = rows_max; box[2] = 1; box[3] = D / 64;
        swz = CU_TENSOR_MAP_SWIZZLE_128B;
    } else {
        rank = 3;
        dims[0] = 32; dims[1] = t->shape[1]; dims[2] = t->shape[0];
        strides[0] = st[1] * 2; strides[1] = st[0] * 2;
        box[0] = 32; box[1] = rows_max; box[2] = 1;
        swz = CU_TENSOR_MAP_SWIZZLE_64B;
    }
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, t->data, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return driver_fail(r, "cuTensorMapEncodeTiled(q)");
    return APD_OK;
}

// ---------------------------------------------------------------- launch
// Self-test settings of the split kernel (the defaults are the product's).
struct SplitTestHooks {
    uint64_t wait_ns = apd::kWaitTimeoutNs;
    int skip_release = 0;  // shared-ring followers never release a stage
    int skip_pfull = 0;    // tensor-core kernel: the softmax warps never hand over P of tile 1
};

// The caller's split_done_event, recorded right after the first kernel of the call.
int record_split_done(const apd_launch_options* opts, cudaStream_t stream) {
    if (!(opts && opts->split_done_event)) return APD_OK;
    // while the stream is being captured into a CUDA graph the record becomes an
    // event-record node (external), so the event still times the replayed kernel
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    cudaError_t e = cudaStreamIsCapturing(stream, &cap);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamIsCapturing");
    e = cudaEventRecordWithFlags(static_cast<cudaEvent_t>(opts->split_done_event), stream,
                                 cap == cudaStreamCaptureStatusActive ? cudaEventRecordExternal : 0u);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventRecord(split_done_event)");
    return APD_OK;
}

// The combine kernel of a call whose first kernel wrote partials (launched with PDL unless
// PDL is off or an event separates the two kernels).
template <int D>
int launch_combine(const Shape& s, const Plan& pl, const apd::CombineParams& cp, cudaStream_t stream,
                   const apd_launch_options* opts) {
    const bool use_pdl = !(opts && opts->disable_pdl);
    cudaLaunchAttribute pdl_attr[1];
    pdl_attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl_attr[0].val.programmaticStreamSerializationAllowed = 1;
    const bool per_unit = combine_per_unit(s, pl);
    const int cw = per_unit ? (s.rows_max >= 8 ? 8 : 4) : combine_warps(s, pl);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = per_unit ? dim3(static_cast<unsigned>(pl.combine_ctas))
                           : dim3(static_cast<unsigned>(s.units), static_cast<unsigned>(s.rows_max));
    cfg.blockDim = dim3(32 * cw);
    cfg.dynamicSmemBytes = per_unit ? 4u * (s.B + 1) : 0u;
    cfg.stream = stream;
    cfg.attrs = pdl_attr;
    cfg.numAttrs = (use_pdl && !(opts && opts->split_done_event)) ? 1 : 0;
    cudaError_t e;
    if (per_unit)
        e = cw == 8 ? cudaLaunchKernelEx(&cfg, apd::combine_unit_kernel<D, 8>, cp)
                    : cudaLaunchKernelEx(&cfg, apd::combine_unit_kernel<D, 4>, cp);
    else
        e = cw == 16 ? cudaLaunchKernelEx(&cfg, apd::combine_kernel<D, 16>, cp)
            : cw == 8 ? cudaLaunchKernelEx(&cfg, apd::combine_kernel<D, 8>, cp)
                      : cudaLaunchKernelEx(&cfg, apd::combine_kernel<D, 4>, cp);
    if (e != cudaSuccess) return cuda_fail(e, "combine_kernel launch");
    return APD_OK;
}

// Mode 3: the tensor-core multi-query kernel, then the combine when units are split and
// not merged in a cluster.
template <int NH>
int launch_mq_tc(const Validated& V, const apd_tensor* q, const apd_tensor* k, const apd_tensor* v,
                 const apd_tensor* pt, const apd_tensor* sl, const apd_tensor* out, float scale, const Plan& pl,
                 void* workspace, DeviceState* dev, cudaStream_t stream, const apd_launch_options* opts,
                 const SplitTestHooks& hooks) {
    constexpr int D = 128;
    using McShape128 = McShapeT<NH>;
    auto kern = apd::decode_mq_tc_kernel<D, NH>;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        const int hi = NH == 64 ? 1 : 0;
        if (!dev->mq_tc_attr_set[hi]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(McShape128::kSmemBytes));
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(decode_mq_tc_kernel)");
            dev->mq_tc_attr_set[hi] = true;
        }
    }
    // K/V boxes of one 64-element block each, so that a tile's rows of one block are
    // contiguous (the canonical operand layout)
    CUtensorMap kmap, vmap;
    int rc = encode_kv_map(&kmap, k, V.kst, D, 1);
    if (!rc) rc = encode_kv_map(&vmap, v, V.vst, D, 1);
    if (rc) return rc;

    const Shape& s = V.s;
    char* ws = static_cast<char*>(workspace);
    apd::McParams mp;
    mp.q = static_cast<const __nv_bfloat16*>(q->data);
    mp.q_sb = V.qst[0];
    mp.q_sh = V.qst[1];
    mp.page_table = pt ? static_cast<const int32_t*>(pt->data) : nullptr;
    mp.pt_s0 = V.pst[0];
    mp.pt_s1 = V.pst[1];
    mp.seq_lens = static_cast<const int32_t*>(sl->data);
    mp.out = static_cast<__nv_bfloat16*>(out->data);
    mp.out_sb = V.ost[0];
    mp.out_sh = V.ost[1];
    mp.o_part = reinterpret_cast<float*>(ws + ws_head_bytes(s));
    mp.ml_part = reinterpret_cast<float*>(ws + ws_head_bytes(s) +
                                          align_up(static_cast<size_t>(pl.slots) * s.rows_max * s.D * 4, kWsAlign));
    mp.flags = reinterpret_cast<uint32_t*>(ws);
    mp.B = s.B;
    mp.Hkv = s.Hkv;
    mp.g = s.g;
    mp.HB = s.HB;
    mp.rows_max = s.rows_max;
    mp.P = V.P;
    mp.NP = V.NP;
    mp.MP = V.MP;
    mp.nhb = pl.hblocks;
    mp.hbh = pl.hb_heads;
    mp.ksplit = pl.ksplit;
    mp.cluster = pl.cluster > 0 ? 1 : 0;
    mp.scale_log2 = scale * 1.4426950408889634f;
    mp.wait_ns = hooks.wait_ns;
    mp.test_skip_pfull = hooks.skip_pfull;

    const bool use_pdl = !(opts && opts->disable_pdl);
    cudaLaunchAttribute attrs[2];
    int na = 0;
    if (pl.cluster > 0) {
        attrs[na].id = cudaLaunchAttributeClusterDimension;
        attrs[na].val.clusterDim.x = static_cast<unsigned>(pl.cluster);
        attrs[na].val.clusterDim.y = 1;
        attrs[na].val.clusterDim.z = 1;
        ++na;
    }
    if (use_pdl) {
        attrs[na].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        attrs[na].val.programmaticStreamSerializationAllowed = 1;
        ++na;
    }
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(pl.ctas));
    cfg.blockDim = dim3(static_cast<unsigned>(McShape128::kThreads));
    cfg.dynamicSmemBytes = McShape128::kSmemBytes;
    cfg.stream = stream;
    cfg.attrs = attrs;
    cfg.numAttrs = na;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, mp, kmap, vmap);
    if (e != cudaSuccess) return cuda_fail(e, "decode_mq_tc_kernel launch");
    rc = record_split_done(opts, stream);
    if (rc) return rc;
    if (pl.combine_ctas > 0) {
        apd::CombineParams cp;
        cp.cum = reinterpret_cast<int32_t*>(ws + kWsAlign);
        cp.seq_lens = mp.seq_lens;
        cp.MP = mp.MP;
        cp.P = mp.P;
        cp.o_part = mp.o_part;
        cp.ml_part = mp.ml_part;
        cp.out = mp.out;
        cp.out_sb = mp.out_sb;
        cp.out_sh = mp.out_sh;
        cp.B = s.B;
        cp.Hkv = s.Hkv;
        cp.g = s.g;
        cp.HB = s.HB;
        cp.rows_max = s.rows_max;
        cp.mode = pl.mode;
        cp.ksplit = pl.ksplit;
        cp.num_workers = pl.workers;
        cp.groups = pl.groups;
        return launch_combine<D>(s, pl, cp, stream, opts);
    }
    return APD_OK;
}

template <int D>
int launch(const Validated& V, const apd_tensor* q, const apd_tensor* k, const apd_tensor* v,
           const apd_tensor* pt, const apd_tensor* sl, const apd_tensor* out, float scale, const Plan& pl,
           void* workspace, DeviceState* dev, cudaStream_t stream, const apd_launch_options* opts,
           const SplitTestHooks& hooks = SplitTestHooks()) {
    if constexpr (D == 128) {
        if (pl.mode == 3)
            return mq_tc_heads(V.s) == 64
                       ? launch_mq_tc<64>(V, q, k, v, pt, sl, out, scale, pl, workspace, dev, stream, opts, hooks)
                       : launch_mq_tc<32>(V, q, k, v, pt, sl, out, scale, pl, workspace, dev, stream, opts, hooks);
    }
    if (pl.mode == 3) return APD_ERR_ARGUMENT;  // planned only for D = 128
    constexpr int kStagesD = kStages<D>;
    // the lean per-tile form everywhere but D = 256 (the split kernel's LEAN parameter lists
    // the measurements)
    constexpr bool kLeanD = D != 256;
    auto kern = apd::split_kernel<D, kStagesD, false, kLeanD>;
    int variant = 0;
    if constexpr (kShareStages<D> > 0) {
        if (pl.share) {
            kern = apd::split_kernel<D, kShareStages<D>, true, kLeanD>;
            variant = 1;
        }
    }
    if (pl.mode != 0) {
        // one CTA per unit (or per split of a unit): the lean per-tile form at D = 32 and 64
        // only (the plain form measured 1% faster for the llama8b shape at D = 128)
        if (pl.mode == 1) kern = apd::unit_kernel<D, kUnitStages<D>, (D == 32 || D == 64), true>;
        else kern = apd::unit_kernel<D, kUnitStages<D>, (D == 32 || D == 64), false>;
        variant = pl.mode == 1 ? 3 : 2;
    }
    const int kSlot = ((D == 32) ? 0 : (D == 64) ? 1 : (D == 128) ? 2 : 3) + 4 * variant;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!dev->smem_attr_set[kSlot]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(kSmemLimit));
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(split_kernel)");
            dev->smem_attr_set[kSlot] = true;
        }
    }
    CUtensorMap kmap, vmap, qmap;
    int rc = encode_kv_map(&kmap, k, V.kst, D);
    if (!rc) rc = encode_kv_map(&vmap, v, V.vst, D);
    if (!rc) rc = encode_q_map(&qmap, q, V.qst, D, V.s.rows_max);
    if (rc) return rc;

    const Shape& s = V.s;
    char* ws = static_cast<char*>(workspace);
    apd::SplitParams sp;
    sp.page_table = pt ? static_cast<const int32_t*>(pt->data) : nullptr;
    sp.pt_s0 = V.pst[0];
    sp.pt_s1 = V.pst[1];
    sp.seq_lens = static_cast<const int32_t*>(sl->data);
    sp.out = static_cast<__nv_bfloat16*>(out->data);
    sp.out_sb = V.ost[0];
    sp.out_sh = V.ost[1];
    sp.flags = reinterpret_cast<uint32_t*>(ws);
    sp.cum_out = reinterpret_cast<int32_t*>(ws + kWsAlign);
    sp.zero_empty = (pl.mode == 0 && pl.combine_ctas == 0) ? 1 : 0;
    sp.o_part = reinterpret_cast<float*>(ws + ws_head_bytes(s));
    sp.ml_part = reinterpret_cast<float*>(ws + ws_head_bytes(s) +
                                          align_up(static_cast<size_t>(pl.slots) * s.rows_max * s.D * 4, kWsAlign));
    sp.B = s.B;
    sp.Hq = s.Hq;
    sp.Hkv = s.Hkv;
    sp.g = s.g;
    sp.HB = s.HB;
    sp.rows_max = s.rows_max;
    sp.P = V.P;
    sp.NP = V.NP;
    sp.MP = V.MP;
    sp.mode = pl.mode;
    sp.ksplit = pl.ksplit;
    sp.num_workers = pl.workers;
    sp.groups = pl.groups;
    sp.warps = pl.warps;
    sp.stage_bytes = stage_bytes(s);
    sp.q_box_bytes = static_cast<uint32_t>(s.rows_max) * s.D * 2u;
    sp.scale_log2 = scale * 1.4426950408889634f;
    sp.wait_ns = hooks.wait_ns;
    sp.test_skip_release = hooks.skip_release;

    // Both kernels are launched with programmatic dependent launch (PDL): each
    // begins launching while the previous kernel in the stream drains, and waits
    // (griddepcontrol.wait) for it before touching global memory.
    const bool use_pdl = !(opts && opts->disable_pdl);
    cudaLaunchAttribute pdl_attr[1];
    pdl_attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl_attr[0].val.programmaticStreamSerializationAllowed = 1;
    {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(static_cast<unsigned>(pl.ctas));
        cfg.blockDim = dim3(static_cast<unsigned>(pl.warps * 32));
        cfg.dynamicSmemBytes = pl.smem;
        cfg.stream = stream;
        cfg.attrs = pdl_attr;
        cfg.numAttrs = use_pdl ? 1 : 0;
        cudaError_t e = cudaLaunchKernelEx(&cfg, kern, sp, kmap, vmap, qmap);
        if (e != cudaSuccess) return cuda_fail(e, "split_kernel launch");
    }
    int rc2 = record_split_done(opts, stream);
    if (rc2) return rc2;
    if (pl.combine_ctas > 0) {
        apd::CombineParams cp;
        cp.cum = sp.cum_out;
        cp.seq_lens = sp.seq_lens;
        cp.MP = sp.MP;
        cp.P = sp.P;
        cp.o_part = sp.o_part;
        cp.ml_part = sp.ml_part;
        cp.out = sp.out;
        cp.out_sb = sp.out_sb;
        cp.out_sh = sp.out_sh;
        cp.B = s.B;
        cp.Hkv = s.Hkv;
        cp.g = s.g;
        cp.HB = s.HB;
        cp.rows_max = s.rows_max;
        cp.mode = pl.mode;
        cp.ksplit = pl.ksplit;
        cp.num_workers = pl.workers;
        cp.groups = pl.groups;
        return launch_combine<D>(s, pl, cp, stream, opts);
    }
    return APD_OK;
}

// ---------------------------------------------------------------- decode projection (GEMV)
constexpr int kGemvStages = 4;
// Warps per CTA, and eighths of the SMs that get a CTA, for the two x paths.  With x staged
// once per CTA (long weight streams), lm_head 100000 x 1536, graph-timed over M = 1..8
// (4 warps on every SM -> 6 warps on 7/8 of them): 56.6 -> 50.1 us at M = 1, 57.6 -> 50.5
// at M = 2, 58.5 -> 51.6 at M = 4, 58.9 -> 52.2 at M = 8; 5 warps on all SMs, 5 warps x 5
// stages, 8 warps x 3 stages all measured between the two.  The shorter streams that load x
// with every stage keep 4 warps on every SM (their stages are 12 KB).
constexpr int gemv_warps(bool xs) { return xs ? 6 : 4; }
constexpr int gemv_sm_eighths(bool xs) { return xs ? 7 : 8; }

// Shared memory of the GEMV kernel: mbarriers, the staged x rows (xs) with a zero chunk,
// alignment, the ring.  x is staged once per CTA when it fits with at least 2 stages.
int gemv_x_pitch(int K) { return 16 * ((K / 8) | 1); }
size_t gemv_smem_bytes(int M, int K, int stages, bool xs, int warps) {
    const size_t x = xs ? static_cast<size_t>(M) * gemv_x_pitch(K) + 16 + 16 : 0;
    return 8ull * warps * stages + 8 + 16 + x + 1024 +
           static_cast<size_t>(warps) * stages * (xs ? apd::kGemvWBytes : apd::kGemvStageBytes);
}
// x is staged once per CTA for long weight streams (W >= 64 MB) when it is at most 32 KB
// (every CTA copies it from L2) and the full ring still fits.  Graph-timed on the
// AstrAI-1B shapes: lm_head (100000 x 1536) 59.3 -> 56.7 us at M = 1, 60.1 -> 58.0 at
// M = 3, 59.7 -> 59.1 at M = 8; the 21 MB layers, which are latency-bound, lose up to
// 3 us to the copy that precedes their first MMA (gate_up M = 8: 8.5 -> 11.8 us).
bool gemv_stage_x(int M, int N, int K) {
    return static_cast<int64_t>(N) * K * 2 >= (64ll << 20) && static_cast<int64_t>(M) * gemv_x_pitch(K) <= 32768 &&
           gemv_smem_bytes(M, K, kGemvStages, true, gemv_warps(true)) <= 232448;
}

// Whole m-tiles per warp when there are between one and four per SM and each is short
// (K <= 2048, at most 64 KB of W per warp): no m-tile is split, every warp writes its
// rows of y directly, and the sum kernel is not launched.  Graph-timed on the AstrAI-1B
// shapes: gate_up (432 m-tiles) 8.5 -> 6.8 us; kv (16 m-tiles, too few warps) went
// 5.9 -> 6.7 us and q (96) was even, so fewer m-tiles than SMs keep the split of units
// over all warps, as do longer rows.
bool gemv_whole_mtiles(int sm_count, int64_t mtiles, int64_t ktiles, bool xs) {
    return mtiles >= sm_count && mtiles <= static_cast<int64_t>(sm_count) * gemv_warps(xs) && ktiles <= 8;
}

int64_t gemv_workers(int sm_count, int64_t mtiles, int64_t ktiles, bool xs) {
    if (gemv_whole_mtiles(sm_count, mtiles, ktiles, xs)) return mtiles;
    const int64_t w = static_cast<int64_t>(sm_count) * gemv_sm_eighths(xs) / 8 * gemv_warps(xs);
    return std::max<int64_t>(1, std::min(w, mtiles * ktiles));
}

// Workspace: [flags 256 B][fp32 partials, 2 per worker].
size_t gemv_ws_bytes(int64_t workers) {
    return kWsAlign + align_up(static_cast<size_t>(2 * workers) * apd::kGemvRows * apd::kGemvXRows * 4, kWsAlign);
}

// One CTA per m-tile for short weight streams (at most 32 MB) with fewer m-tiles than SMs
// and at least two k-tiles: up to 4 warps split the m-tile's k-tiles and add their parts
// in shared memory, so the call is one kernel with no partials in global memory.
bool gemv_cta_per_mtile(int sm_count, int M, int N, int K, int64_t mtiles, int64_t ktiles) {
    return !gemv_stage_x(M, N, K) && mtiles <= sm_count && ktiles >= 2 &&
           static_cast<int64_t>(N) * K * 2 <= (32ll << 20);
}

// The launch of one GEMV shape, as apd_gemv_bf16 makes it.
struct GemvLaunch {
    bool xs, whole, cta;
    int warps;
    int64_t workers, ctas, sum_ctas;
    size_t smem, ws_bytes;
};
GemvLaunch gemv_launch(int sm_count, int M, int N, int K) {
    GemvLaunch L;
    const int64_t mtiles = (static_cast<int64_t>(N) + apd::kGemvRows - 1) / apd::kGemvRows;
    const int64_t ktiles = (static_cast<int64_t>(K) + apd::kGemvCols - 1) / apd::kGemvCols;
    L.xs = gemv_stage_x(M, N, K);
    L.cta = gemv_cta_per_mtile(sm_count, M, N, K, mtiles, ktiles);
    if (L.cta) {
        L.whole = false;
        L.warps = static_cast<int>(std::min<int64_t>(4, ktiles));
        L.workers = mtiles * L.warps;
        L.ctas = mtiles;
        L.sum_ctas = 0;
        L.ws_bytes = gemv_ws_bytes(0);
    } else {
        L.warps = gemv_warps(L.xs);
        L.whole = gemv_whole_mtiles(sm_count, mtiles, ktiles, L.xs);
        L.workers = gemv_workers(sm_count, mtiles, ktiles, L.xs);
        // whole m-tiles per warp: as few warps per CTA as put every SM to work (gate_up,
        // 432 m-tiles: 3 warps on 144 SMs instead of 4 on 108, 6.82 -> 6.59 us)
        if (L.whole) L.warps = static_cast<int>(std::min<int64_t>(L.warps, (mtiles + sm_count - 1) / sm_count));
        L.ctas = (L.workers + L.warps - 1) / L.warps;
        L.sum_ctas = L.whole ? 0 : (mtiles + 3) / 4;
        L.ws_bytes = gemv_ws_bytes(L.workers);
    }
    L.smem = gemv_smem_bytes(M, K, kGemvStages, L.xs, L.warps);
    return L;
}

// A bf16 row-major matrix [rows, K]: K contiguous, row stride a multiple of 8
// elements, base 16-byte aligned (the TMA rules for the tiled loads).
bool gemv_matrix_ok(const apd_tensor* t, int64_t* ld) {
    int64_t st[2];
    normalized_strides(t, st);
    if (st[1] != 1 || st[0] <= 0 || st[0] % 8 != 0 || st[0] * 2 >= (1ll << 40)) return false;
    if (reinterpret_cast<uintptr_t>(t->data) & 15u) return false;
    *ld = st[0];
    return true;
}

int encode_gemv_map(CUtensorMap* map, const apd_tensor* t, int64_t ld, int box_rows) {
    auto fn = encode_fn();
    if (!fn) return driver_fail(-1, "cuTensorMapEncodeTiled entry point");
    cuuint64_t dims[2] = {static_cast<cuuint64_t>(t->shape[1]), static_cast<cuuint64_t>(t->shape[0])};
    cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
    cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, t->data, dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) return driver_fail(r, "cuTensorMapEncodeTiled(gemv)");
    return APD_OK;
}

struct GemvShape {
    int M, N, K;
    int64_t ldx, ldw, ysm, ysn, units, mtiles, ktiles;
};

int gemv_validate(const apd_tensor* x, const apd_tensor* w, const apd_tensor* y, GemvShape* g) {
    if (!x || !w || !y) return APD_ERR_NULL_POINTER;
    if (x->dtype != APD_DTYPE_BF16 || w->dtype != APD_DTYPE_BF16 || y->dtype != APD_DTYPE_BF16) return APD_ERR_DTYPE;
    if (x->ndim != 2 || w->ndim != 2 || y->ndim != 2) return APD_ERR_SHAPE;
    const int64_t M = x->shape[0], K = x->shape[1], N = w->shape[0];
    if (w->shape[1] != K || y->shape[0] != M || y->shape[1] != N) return APD_ERR_SHAPE;
    if (M < 1 || M > APD_GEMV_MAX_M || N < 1 || K < 1) return APD_ERR_SHAPE;
    if (N > INT32_MAX / 2 || K > INT32_MAX / 2) return APD_ERR_TOO_LARGE;
    if (is_null(x) || is_null(w) || is_null(y)) return APD_ERR_NULL_POINTER;
    if (K % 8 != 0) return APD_ERR_LAYOUT;
    if (!gemv_matrix_ok(x, &g->ldx) || !gemv_matrix_ok(w, &g->ldw)) return APD_ERR_LAYOUT;
    int64_t yst[2];
    normalized_strides(y, yst);
    if (yst[0] < 0 || yst[1] < 0 || (reinterpret_cast<uintptr_t>(y->data) & 1u)) return APD_ERR_LAYOUT;
    g->M = static_cast<int>(M);
    g->N = static_cast<int>(N);
    g->K = static_cast<int>(K);
    g->ysm = yst[0];
    g->ysn = yst[1];
    g->mtiles = (N + apd::kGemvRows - 1) / apd::kGemvRows;
    g->ktiles = (K + apd::kGemvCols - 1) / apd::kGemvCols;
    g->units = g->mtiles * g->ktiles;
    return APD_OK;
}

// ---------------------------------------------------------------- multi-query (prefill)
int prefill_stages(int D) { return D == 32 ? 8 : D == 64 ? 6 : D == 128 ? 4 : 3; }

// Default prefill kernel: the tcgen05 one for every head dim (mma.sync stays selectable).
constexpr bool kPrefillAutoTc = true;

size_t prefill_smem_bytes(int D) {
    return 16ull * prefill_stages(D) + 8 + 1024 + static_cast<size_t>(prefill_stages(D)) * 2 * apd::kTile * D * 2;
}

struct PrefillCheck {
    Validated V;  // the KV side, checked as for decode (q's role taken by a [B, Hq, D] view)
    int Lq;
    int64_t qst[4], ost[4], mst[3];
    int mask_dims;
};

int prefill_validate(const apd_tensor* q, const apd_tensor* k, const apd_tensor* v, const apd_tensor* pt,
                     const apd_tensor* sl, const apd_tensor* mask, const apd_tensor* out, int causal_offset,
                     PrefillCheck* C) {
    if (!q || !out || !pt) return APD_ERR_NULL_POINTER;
    if (q->dtype != APD_DTYPE_BF16 || out->dtype != APD_DTYPE_BF16) return APD_ERR_DTYPE;
    if (q->ndim != 4 || out->ndim != 4) return APD_ERR_SHAPE;
    for (int i = 0; i < 4; ++i)
        if (q->shape[i] != out->shape[i] || q->shape[i] < 0) return APD_ERR_SHAPE;
    if (q->shape[1] < 1 || q->shape[1] > (1 << 20)) return APD_ERR_SHAPE;
    if (causal_offset < -1) return APD_ERR_ARGUMENT;
    // the KV side and the per-sequence tensors: reuse the decode checks on [B, Hq, D] views
    apd_tensor q3 = *q, o3 = *out;
    q3.ndim = o3.ndim = 3;
    q3.shape[1] = q->shape[2];
    q3.shape[2] = q->shape[3];
    q3.stride[1] = q->stride[2];
    q3.stride[2] = q->stride[3];
    o3.shape[1] = out->shape[2];
    o3.shape[2] = out->shape[3];
    o3.stride[1] = out->stride[2];
    o3.stride[2] = out->stride[3];
    int rc = validate(&q3, k, v, pt, sl, &o3, 0, &C->V);
    if (rc) return rc;
    C->Lq = static_cast<int>(q->shape[1]);
    if (static_cast<int64_t>(C->Lq) * C->V.s.g > (1 << 26)) return APD_ERR_TOO_LARGE;
    if (C->V.s.B > 0 && (!aligned_bf16_layout(q, C->qst) || !aligned_bf16_layout(out, C->ost))) return APD_ERR_LAYOUT;
    C->mask_dims = 0;
    C->mst[0] = C->mst[1] = C->mst[2] = 0;
    if (mask) {
        if (mask->dtype != APD_DTYPE_UINT8) return APD_ERR_DTYPE;
        if (mask->ndim != 2 && mask->ndim != 3) return APD_ERR_SHAPE;
        if (mask->shape[0] != q->shape[0]) return APD_ERR_SHAPE;
        if (mask->ndim == 3 && mask->shape[1] != q->shape[1]) return APD_ERR_SHAPE;
        // every key index below the page-table capacity must be inside the mask
        if (mask->shape[mask->ndim - 1] < static_cast<int64_t>(C->V.MP) * C->V.P) return APD_ERR_SHAPE;
        if (C->V.s.B > 0 && is_null(mask)) return APD_ERR_NULL_POINTER;
        int64_t st[3];
        normalized_strides(mask, st);
        for (int i = 0; i < mask->ndim; ++i)
            if (st[i] < 0) return APD_ERR_LAYOUT;
        C->mst[0] = st[0];
        C->mst[1] = mask->ndim == 3 ? st[1] : 0;
        C->mst[2] = st[mask->ndim - 1];
        C->mask_dims = mask->ndim;
    }
    return APD_OK;
}

apd::PrefillParams prefill_params(const PrefillCheck& C, const apd_tensor* q, const apd_tensor* pt,
                                  const apd_tensor* sl, const apd_tensor* mask, const apd_tensor* out, float scale,
                                  int causal_offset, int rows_per_cta) {
    const Shape& s = C.V.s;
    apd::PrefillParams pp;
    pp.q = static_cast<const __nv_bfloat16*>(q->data);
    pp.q_sb = C.qst[0];
    pp.q_si = C.qst[1];
    pp.q_sh = C.qst[2];
    pp.out = static_cast<__nv_bfloat16*>(out->data);
    pp.o_sb = C.ost[0];
    pp.o_si = C.ost[1];
    pp.o_sh = C.ost[2];
    pp.page_table = static_cast<const int32_t*>(pt->data);
    pp.pt_s0 = C.V.pst[0];
    pp.pt_s1 = C.V.pst[1];
    pp.seq_lens = static_cast<const int32_t*>(sl->data);
    pp.mask = mask ? static_cast<const uint8_t*>(mask->data) : nullptr;
    pp.m_sb = C.mst[0];
    pp.m_si = C.mst[1];
    pp.m_st = C.mst[2];
    pp.flags = nullptr;
    pp.B = s.B;
    pp.Lq = C.Lq;
    pp.Hq = s.Hq;
    pp.Hkv = s.Hkv;
    pp.g = s.g;
    pp.P = C.V.P;
    pp.NP = C.V.NP;
    pp.MP = C.V.MP;
    pp.blocks_per_head =
        static_cast<int32_t>((static_cast<int64_t>(C.Lq) * s.g + rows_per_cta - 1) / rows_per_cta);
    pp.causal_offset = causal_offset;
    pp.scale_log2 = scale * 1.4426950408889634f;
    return pp;
}

template <typename Kernel>
int launch_prefill_grid(Kernel kern, const apd::PrefillParams& pp, const CUtensorMap& kmap, const CUtensorMap& vmap,
                        int threads, size_t smem, cudaStream_t stream, const char* what) {
    const int64_t grid = static_cast<int64_t>(pp.B) * pp.Hkv * pp.blocks_per_head;
    if (grid > INT32_MAX) return APD_ERR_TOO_LARGE;
    cudaLaunchAttribute pdl_attr[1];
    pdl_attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl_attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cfg.attrs = pdl_attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, pp, kmap, vmap);
    if (e != cudaSuccess) return cuda_fail(e, what);
    return APD_OK;
}

// mma.sync kernel (every head dim)
template <int D>
int launch_prefill(const PrefillCheck& C, const apd_tensor* q, const apd_tensor* k, const apd_tensor* v,
                   const apd_tensor* pt, const apd_tensor* sl, const apd_tensor* mask, const apd_tensor* out,
                   float scale, int causal_offset, DeviceState* dev, cudaStream_t stream) {
    constexpr int kStages = (D == 32) ? 8 : (D == 64) ? 6 : (D == 128) ? 4 : 3;
    auto kern = apd::prefill_kernel<D, kStages>;
    constexpr int kSlot = (D == 32) ? 0 : (D == 64) ? 1 : (D == 128) ? 2 : 3;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!dev->prefill_attr_set[kSlot]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(prefill_smem_bytes(D)));
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefill_kernel)");
            dev->prefill_attr_set[kSlot] = true;
        }
    }
    CUtensorMap kmap, vmap;
    int rc = encode_kv_map(&kmap, k, C.V.kst, D);
    if (!rc) rc = encode_kv_map(&vmap, v, C.V.vst, D);
    if (rc) return rc;
    const apd::PrefillParams pp =
        prefill_params(C, q, pt, sl, mask, out, scale, causal_offset, apd::PrefillShape<D>::kRows);
    return launch_prefill_grid(kern, pp, kmap, vmap, apd::PrefillShape<D>::kThreads, prefill_smem_bytes(D), stream,
                               "prefill_kernel launch");
}

// tcgen05 kernel with two 128-row Q tiles per CTA (D = 32, 64, 128)
template <int D>
int launch_prefill_tc2(const PrefillCheck& C, const apd_tensor* q, const apd_tensor* k, const apd_tensor* v,
                       const apd_tensor* pt, const apd_tensor* sl, const apd_tensor* mask, const apd_tensor* out,
                       float scale, int causal_offset, DeviceState* dev, cudaStream_t stream) {
    using T = apd::Tc2Shape<D>;
    auto kern = apd::prefill_tc2_kernel<D>;
    constexpr int kSlot = (D == 32) ? 0 : (D == 64) ? 1 : 2;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!dev->prefill_tc2_attr_set[kSlot]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(T::kSmemBytes));
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefill_tc2_kernel)");
            dev->prefill_tc2_attr_set[kSlot] = true;
        }
    }
    CUtensorMap kmap, vmap;
    int rc = encode_kv_map(&kmap, k, C.V.kst, D, 1);
    if (!rc) rc = encode_kv_map(&vmap, v, C.V.vst, D, 1);
    if (rc) return rc;
    const apd::PrefillParams pp = prefill_params(C, q, pt, sl, mask, out, scale, causal_offset, 2 * T::kM);
    return launch_prefill_grid(kern, pp, kmap, vmap, T::kThreads, T::kSmemBytes, stream, "prefill_tc2_kernel launch");
}

// tcgen05 kernel, one 128-row Q tile per CTA (every D)
template <int D>
int launch_prefill_tc(const PrefillCheck& C, const apd_tensor* q, const apd_tensor* k, const apd_tensor* v,
                      const apd_tensor* pt, const apd_tensor* sl, const apd_tensor* mask, const apd_tensor* out,
                      float scale, int causal_offset, DeviceState* dev, cudaStream_t stream) {
    using T = apd::TcShape<D>;
    auto kern = apd::prefill_tc_kernel<D>;
    constexpr int kSlot = (D == 32) ? 0 : (D == 64) ? 1 : (D == 128) ? 2 : 3;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!dev->prefill_tc_attr_set[kSlot]) {
            cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(T::kSmemBytes));
            if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(prefill_tc_kernel)");
            dev->prefill_tc_attr_set[kSlot] = true;
        }
    }
    CUtensorMap kmap, vmap;
    int rc = encode_kv_map(&kmap, k, C.V.kst, D, 1);
    if (!rc) rc = encode_kv_map(&vmap, v, C.V.vst, D, 1);
    if (rc) return rc;
    const apd::PrefillParams pp = prefill_params(C, q, pt, sl, mask, out, scale, causal_offset, T::kM);
    return launch_prefill_grid(kern, pp, kmap, vmap, T::kThreads, T::kSmemBytes, stream, "prefill_tc_kernel launch");
}

// ---------------------------------------------------------------- built-in scratch
// Scratch of apd_attn_paged_decode_noalloc: a static device array, so that entry
// point allocates nothing.  Host code must not use its name as an address (on the
// host it is only a stand-in); the device address comes from cudaGetSymbolAddress.
static __device__ __align__(256) uint8_t g_noalloc_scratch[APD_NOALLOC_SCRATCH_BYTES];

void* g_noalloc_scratch_addr[128] = {};

// Device address of g_noalloc_scratch on the current device, looked up once per device.
int noalloc_scratch(void** out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    if (dev < 0 || dev >= 128) return APD_ERR_ARGUMENT;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_noalloc_scratch_addr[dev]) {
        void* ptr = nullptr;
        e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
        if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(noalloc scratch)");
        g_noalloc_scratch_addr[dev] = ptr;
    }
    *out = g_noalloc_scratch_addr[dev];
    return APD_OK;
}

}  // namespace

extern "C" {

size_t apd_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim, int num_splits) {
    Shape s;
    if (make_shape(batch, num_q_heads, num_kv_heads, head_dim, &s) != APD_OK) return 0;
    if (num_splits < 0) return 0;
    int sm_count = kDefaultSmCount;
    int dev = 0;
    if (num_splits == 0 && cudaGetDevice(&dev) == cudaSuccess) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0) sm_count = n;
    }
    cudaGetLastError();  // a missing device is not an error of this query
    Plan pl;
    if (make_plan(s, num_splits, sm_count, SIZE_MAX, -1, &pl) != APD_OK) return 0;
    return pl.ws_needed;
}

int apd_workspace_init(void* workspace, size_t workspace_bytes, apd_stream_t stream) {
    if (!workspace) return APD_ERR_NULL_POINTER;
    if (workspace_bytes < kWsAlign || (reinterpret_cast<uintptr_t>(workspace) % kWsAlign)) return APD_ERR_WORKSPACE;
    cudaError_t e = cudaMemsetAsync(workspace, 0, workspace_bytes, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(workspace)");
    return APD_OK;
}

}  // extern "C"

namespace {

// The decode call behind every workspace entry point; page_table == nullptr is the
// contiguous-KV form (see validate).
int decode_impl(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* out, float scale,
                int num_splits, void* workspace, size_t workspace_bytes, apd_stream_t stream,
                const apd_launch_options* options, const SplitTestHooks* hooks = nullptr) {
    if (options && options->reserved != 0) return APD_ERR_ARGUMENT;
    Validated V;
    int rc = validate(q, k_cache, v_cache, page_table, seq_lens, out, num_splits, &V);
    if (rc) return rc;
    if (!workspace) return APD_ERR_WORKSPACE;
    if (reinterpret_cast<uintptr_t>(workspace) % kWsAlign) return APD_ERR_WORKSPACE;
    if (V.s.B == 0) return APD_OK;
    Plan pl;
    const int64_t tiles_bound = V.s.units * V.MP * ((V.P + apd::kTile - 1) / apd::kTile);
    // A fixed split count does not depend on the device: check its workspace
    // before any CUDA call.
    if (num_splits > 0) {
        rc = make_plan(V.s, num_splits, kDefaultSmCount, workspace_bytes, tiles_bound, &pl);
        if (rc) return rc;
    }
    DeviceState* dev = nullptr;
    rc = device_state(&dev);
    if (rc) return rc;
    const SplitTestHooks h = hooks ? *hooks : SplitTestHooks();
    rc = make_plan(V.s, num_splits, dev->sm_count, workspace_bytes, tiles_bound, &pl,
                   options ? options->host_seq_lens : nullptr, static_cast<int64_t>(V.MP) * V.P,
                   /*allow_tc=*/!h.skip_release, mq_cluster_caps(dev));
    if (rc) return rc;
    // the release self-test needs the shared K/V ring (auto splits, more than 16 q heads per kv head)
    if (h.skip_release && !pl.share) return APD_ERR_ARGUMENT;
    // the stall self-test needs the tensor-core multi-query kernel
    if (h.skip_pfull && pl.mode != 3) return APD_ERR_ARGUMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    switch (V.s.D) {
        case 32: return launch<32>(V, q, k_cache, v_cache, page_table, seq_lens, out, scale, pl, workspace, dev, st, options, h);
        case 64: return launch<64>(V, q, k_cache, v_cache, page_table, seq_lens, out, scale, pl, workspace, dev, st, options, h);
        case 128: return launch<128>(V, q, k_cache, v_cache, page_table, seq_lens, out, scale, pl, workspace, dev, st, options, h);
        case 256: return launch<256>(V, q, k_cache, v_cache, page_table, seq_lens, out, scale, pl, workspace, dev, st, options, h);
        default: return APD_ERR_HEAD_DIM;
    }
}

}  // namespace

extern "C" {

int apd_attn_paged_decode_ex(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                             const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* out,
                             float scale, int num_splits, void* workspace, size_t workspace_bytes,
                             apd_stream_t stream, const apd_launch_options* options) {
    if (!page_table) return APD_ERR_NULL_POINTER;
    return decode_impl(q, k_cache, v_cache, page_table, seq_lens, out, scale, num_splits, workspace, workspace_bytes,
                       stream, options);
}

int apd_attn_paged_decode(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                          const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* out,
                          float scale, int num_splits, void* workspace, size_t workspace_bytes,
                          apd_stream_t stream) {
    return apd_attn_paged_decode_ex(q, k_cache, v_cache, page_table, seq_lens, out, scale, num_splits, workspace,
                                    workspace_bytes, stream, nullptr);
}

int apd_attn_contig_decode_ex(const apd_tensor* q, const apd_tensor* k, const apd_tensor* v,
                              const apd_tensor* seq_lens, const apd_tensor* out, float scale, int num_splits,
                              void* workspace, size_t workspace_bytes, apd_stream_t stream,
                              const apd_launch_options* options) {
    return decode_impl(q, k, v, nullptr, seq_lens, out, scale, num_splits, workspace, workspace_bytes, stream,
                       options);
}

int apd_attn_contig_decode(const apd_tensor* q, const apd_tensor* k, const apd_tensor* v, const apd_tensor* seq_lens,
                           const apd_tensor* out, float scale, int num_splits, void* workspace,
                           size_t workspace_bytes, apd_stream_t stream) {
    return decode_impl(q, k, v, nullptr, seq_lens, out, scale, num_splits, workspace, workspace_bytes, stream,
                       nullptr);
}

int apd_attn_paged_decode_noalloc(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                                  const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* out,
                                  float scale, int num_splits, apd_stream_t stream) {
    if (!page_table) return APD_ERR_NULL_POINTER;
    Validated V;
    int rc = validate(q, k_cache, v_cache, page_table, seq_lens, out, num_splits, &V);
    if (rc) return rc;
    if (V.s.B == 0) return APD_OK;
    constexpr size_t kScratch = APD_NOALLOC_SCRATCH_BYTES;
    Plan pl;
    const int64_t tiles_bound = V.s.units * V.MP * ((V.P + apd::kTile - 1) / apd::kTile);
    if (num_splits > 0) {
        rc = make_plan(V.s, num_splits, kDefaultSmCount, kScratch, tiles_bound, &pl);
        if (rc == APD_ERR_WORKSPACE) return APD_ERR_SCRATCH_LIMIT;
        if (rc) return rc;
    }
    DeviceState* dev = nullptr;
    rc = device_state(&dev);
    if (rc) return rc;
    rc = make_plan(V.s, num_splits, dev->sm_count, kScratch, tiles_bound, &pl, nullptr, 0, true,
                   mq_cluster_caps(dev));
    if (rc == APD_ERR_WORKSPACE) return APD_ERR_SCRATCH_LIMIT;
    if (rc) return rc;
    void* scratch = nullptr;
    rc = noalloc_scratch(&scratch);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    switch (V.s.D) {
        case 32: return launch<32>(V, q, k_cache, v_cache, page_table, seq_lens, out, scale, pl, scratch, dev, st, nullptr);
        case 64: return launch<64>(V, q, k_cache, v_cache, page_table, seq_lens, out, scale, pl, scratch, dev, st, nullptr);
        case 128: return launch<128>(V, q, k_cache, v_cache, page_table, seq_lens, out, scale, pl, scratch, dev, st, nullptr);
        case 256: return launch<256>(V, q, k_cache, v_cache, page_table, seq_lens, out, scale, pl, scratch, dev, st, nullptr);
        default: return APD_ERR_HEAD_DIM;
    }
}

int apd_attn_paged_prefill(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                           const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* mask,
                           const apd_tensor* out, float scale, int causal_offset, apd_stream_t stream) {
    return apd_attn_paged_prefill_ex(q, k_cache, v_cache, page_table, seq_lens, mask, out, scale, causal_offset,
                                     stream, APD_PREFILL_AUTO);
}

int apd_attn_paged_prefill_ex(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                              const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* mask,
                              const apd_tensor* out, float scale, int causal_offset, apd_stream_t stream,
                              int kernel) {
    if (kernel != APD_PREFILL_AUTO && kernel != APD_PREFILL_MMA_SYNC && kernel != APD_PREFILL_TCGEN05)
        return APD_ERR_ARGUMENT;
    PrefillCheck C;
    int rc = prefill_validate(q, k_cache, v_cache, page_table, seq_lens, mask, out, causal_offset, &C);
    if (rc) return rc;
    const int D = C.V.s.D;
    const bool tc = kernel == APD_PREFILL_TCGEN05 || (kernel == APD_PREFILL_AUTO && kPrefillAutoTc);
    if (C.V.s.B == 0) return APD_OK;
    DeviceState* dev = nullptr;
    rc = device_state(&dev);
    if (rc) return rc;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    // two Q tiles per CTA when a kv head has more than one tile of query rows
    const bool two_tiles = static_cast<int64_t>(C.Lq) * C.V.s.g > 128;
    if (tc && two_tiles && D == 32)
        return launch_prefill_tc2<32>(C, q, k_cache, v_cache, page_table, seq_lens, mask, out, scale, causal_offset, dev, st);
    if (tc && two_tiles && D == 64)
        return launch_prefill_tc2<64>(C, q, k_cache, v_cache, page_table, seq_lens, mask, out, scale, causal_offset, dev, st);
    if (tc && two_tiles && D == 128)
        return launch_prefill_tc2<128>(C, q, k_cache, v_cache, page_table, seq_lens, mask, out, scale, causal_offset, dev, st);
    if (tc) {
        switch (D) {
            case 32: return launch_prefill_tc<32>(C, q, k_cache, v_cache, page_table, seq_lens, mask, out, scale, causal_offset, dev, st);
            case 64: return launch_prefill_tc<64>(C, q, k_cache, v_cache, page_table, seq_lens, mask, out, scale, causal_offset, dev, st);
            case 128: return launch_prefill_tc<128>(C, q, k_cache, v_cache, page_table, seq_lens, mask, out, scale, causal_offset, dev, st);
            case 256: return launch_prefill_tc<256>(C, q, k_cache, v_cache, page_table, seq_lens, mask, out, scale, causal_offset, dev, st);
            default: return APD_ERR_HEAD_DIM;
        }
    }
    switch (D) {
        case 32: return launch_prefill<32>(C, q, k_cache, v_cache, page_table, seq_lens, mask, out, scale, causal_offset, dev, st);
        case 64: return launch_prefill<64>(C, q, k_cache, v_cache, page_table, seq_lens, mask, out, scale, causal_offset, dev, st);
        case 128: return launch_prefill<128>(C, q, k_cache, v_cache, page_table, seq_lens, mask, out, scale, causal_offset, dev, st);
        case 256: return launch_prefill<256>(C, q, k_cache, v_cache, page_table, seq_lens, mask, out, scale, causal_offset, dev, st);
        default: return APD_ERR_HEAD_DIM;
    }
}

int apd_gemv_query_plan(int m, int n, int k, int sm_count, apd_gemv_plan* plan) {
    if (!plan) return APD_ERR_NULL_POINTER;
    if (m < 1 || m > APD_GEMV_MAX_M || n < 1 || k < 1) return APD_ERR_ARGUMENT;
    if (sm_count <= 0) {
        DeviceState* dev = nullptr;
        const int rc = device_state(&dev);
        if (rc) return rc;
        sm_count = dev->sm_count;
    }
    const GemvLaunch L = gemv_launch(sm_count, m, n, k);
    plan->workers = static_cast<int32_t>(L.workers);
    plan->grid_ctas = static_cast<int32_t>(L.ctas);
    plan->warps_per_cta = L.warps;
    plan->stages = kGemvStages;
    plan->x_staged = L.xs ? 1 : 0;
    plan->sum_ctas = static_cast<int32_t>(L.sum_ctas);
    plan->cta_per_mtile = L.cta ? 1 : 0;
    plan->workspace_bytes = static_cast<int64_t>(L.ws_bytes);
    return APD_OK;
}

size_t apd_gemv_workspace_size(int m, int n, int k) {
    if (m < 1 || m > APD_GEMV_MAX_M || n < 1 || k < 1) return 0;
    int sm_count = kDefaultSmCount;
    int dev = 0;
    if (cudaGetDevice(&dev) == cudaSuccess) {
        int c = 0;
        if (cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && c > 0) sm_count = c;
    }
    cudaGetLastError();
    return gemv_launch(sm_count, m, n, k).ws_bytes;
}

int apd_gemv_bf16(const apd_tensor* x, const apd_tensor* w, const apd_tensor* y, void* workspace,
                  size_t workspace_bytes, apd_stream_t stream) {
    GemvShape g;
    int rc = gemv_validate(x, w, y, &g);
    if (rc) return rc;
    if (!workspace || (reinterpret_cast<uintptr_t>(workspace) % kWsAlign)) return APD_ERR_WORKSPACE;
    DeviceState* dev = nullptr;
    rc = device_state(&dev);
    if (rc) return rc;
    const GemvLaunch L = gemv_launch(dev->sm_count, g.M, g.N, g.K);
    if (workspace_bytes < L.ws_bytes) return APD_ERR_WORKSPACE;
    auto kern = L.xs ? apd::gemv_kernel<kGemvStages, true> : apd::gemv_kernel<kGemvStages, false>;
    {
        std::lock_guard<std::mutex> lock(g_mu);
        if (!dev->gemv_attr_set) {  // the largest either variant uses, for both
            for (auto k : {apd::gemv_kernel<kGemvStages, true>, apd::gemv_kernel<kGemvStages, false>}) {
                cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 232448);
                if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(gemv_kernel)");
            }
            dev->gemv_attr_set = true;
        }
    }
    CUtensorMap wmap, xmap;
    rc = encode_gemv_map(&wmap, w, g.ldw, apd::kGemvRows);
    if (!rc) rc = encode_gemv_map(&xmap, x, g.ldx, apd::kGemvXRows);
    if (rc) return rc;
    apd::GemvParams gp;
    gp.x = static_cast<const __nv_bfloat16*>(x->data);
    gp.ldx = g.ldx;
    gp.x_pitch = gemv_x_pitch(g.K);
    gp.y = static_cast<__nv_bfloat16*>(y->data);
    gp.y_sm = g.ysm;
    gp.y_sn = g.ysn;
    gp.flags = static_cast<uint32_t*>(workspace);
    gp.part = reinterpret_cast<float*>(static_cast<char*>(workspace) + kWsAlign);
    gp.M = g.M;
    gp.N = g.N;
    gp.K = g.K;
    gp.mtiles = static_cast<int32_t>(g.mtiles);
    gp.ktiles = static_cast<int32_t>(g.ktiles);
    gp.num_workers = static_cast<int32_t>(L.workers);
    gp.warps = L.warps;
    gp.cta_per_mtile = L.cta ? 1 : 0;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaLaunchAttribute pdl_attr[1];
    pdl_attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    pdl_attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(L.ctas));
    cfg.blockDim = dim3(32 * L.warps);
    cfg.dynamicSmemBytes = L.smem;
    cfg.stream = st;
    cfg.attrs = pdl_attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaLaunchKernelEx(&cfg, kern, gp, wmap, xmap);
    if (e != cudaSuccess) return cuda_fail(e, "gemv_kernel launch");
    cudaLaunchConfig_t cfg2 = {};
    cfg2.gridDim = dim3(static_cast<unsigned>(L.sum_ctas));
    cfg2.blockDim = dim3(128);
    cfg2.stream = st;
    cfg2.attrs = pdl_attr;
    cfg2.numAttrs = 1;
    if (L.sum_ctas > 0) {  // some m-tiles are shared by warps of different CTAs: add their partials
        e = cudaLaunchKernelEx(&cfg2, apd::gemv_sum_kernel, gp);
        if (e != cudaSuccess) return cuda_fail(e, "gemv_sum_kernel launch");
    }
    return APD_OK;
}

int apd_read_device_flags(const void* workspace, size_t workspace_bytes, apd_stream_t stream, uint32_t* flags,
                          int clear) {
    if (!workspace || !flags) return APD_ERR_NULL_POINTER;
    if (workspace_bytes < kWsAlign) return APD_ERR_WORKSPACE;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaStreamSynchronize(st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
    e = cudaMemcpy(flags, workspace, sizeof(uint32_t), cudaMemcpyDeviceToHost);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(flags)");
    if (clear) {
        e = cudaMemset(const_cast<void*>(workspace), 0, sizeof(uint32_t));
        if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(flags)");
    }
    return APD_OK;
}

int apd_query_plan(int batch, int num_q_heads, int num_kv_heads, int head_dim, int num_splits,
                   size_t workspace_bytes, int sm_count, apd_plan* plan) {
    return apd_query_plan_ex(batch, num_q_heads, num_kv_heads, head_dim, num_splits, workspace_bytes, sm_count,
                             nullptr, 0, plan);
}

int apd_query_plan_ex(int batch, int num_q_heads, int num_kv_heads, int head_dim, int num_splits,
                      size_t workspace_bytes, int sm_count, const int32_t* host_seq_lens, int64_t max_seq_len,
                      apd_plan* plan) {
    if (!plan) return APD_ERR_NULL_POINTER;
    if (host_seq_lens && max_seq_len < 0) return APD_ERR_ARGUMENT;
    Shape s;
    int rc = make_shape(batch, num_q_heads, num_kv_heads, head_dim, &s);
    if (rc) return rc;
    const McCaps* caps = nullptr;
    if (sm_count <= 0) {
        DeviceState* dev = nullptr;
        rc = device_state(&dev);
        if (rc) return rc;
        sm_count = dev->sm_count;
        caps = mq_cluster_caps(dev);
    }
    Plan pl;
    rc = make_plan(s, num_splits, sm_count, workspace_bytes, -1, &pl, host_seq_lens, max_seq_len, true, caps);
    if (rc) return rc;
    plan->mode = pl.mode;
    plan->num_workers = pl.workers;
    plan->grid_ctas = pl.ctas;
    plan->warps_per_cta = pl.warps;
    plan->stages = pl.stages;
    plan->rows_per_unit = s.rows_max;
    plan->head_blocks = s.HB;
    plan->combine_ctas = pl.combine_ctas;
    plan->smem_bytes = static_cast<int64_t>(pl.smem);
    plan->partial_slots = pl.slots;
    plan->workspace_bytes = static_cast<int64_t>(pl.ws_needed);
    plan->shared_kv_ring = pl.share ? 1 : 0;
    plan->cluster_size = pl.cluster;
    plan->q_head_blocks = pl.mode == 3 ? pl.hblocks : 1;
    plan->q_heads_per_block = pl.mode == 3 ? pl.hb_heads : 0;
    return APD_OK;
}

const char* apd_status_string(int status) {
    switch (status) {
        case APD_OK: return "ok";
        case APD_ERR_NULL_POINTER: return "a tensor descriptor or its data pointer is NULL";
        case APD_ERR_DTYPE: return "wrong dtype: q/k_cache/v_cache/out must be bf16, page_table/seq_lens int32";
        case APD_ERR_SHAPE: return "tensor ranks or extents disagree";
        case APD_ERR_GQA: return "num_q_heads must be a multiple of num_kv_heads";
        case APD_ERR_HEAD_DIM: return "head_dim must be 32, 64, 128 or 256";
        case APD_ERR_LAYOUT:
            return "layout: the head dim must be contiguous and other strides / base pointers 16-byte aligned "
                   "(seq_lens contiguous)";
        case APD_ERR_PAGE_SIZE: return "page_size must be a positive multiple of 32";
        case APD_ERR_NUM_SPLITS: return "num_splits must be >= 0";
        case APD_ERR_WORKSPACE: return "workspace is NULL, not 256-byte aligned, or smaller than apd_workspace_size()";
        case APD_ERR_TOO_LARGE: return "problem too large (batch > APD_MAX_BATCH or index overflow)";
        case APD_ERR_CUDA: return "a CUDA call failed (see apd_last_cuda_error)";
        case APD_ERR_ARGUMENT: return "invalid argument";
        case APD_ERR_SCRATCH_LIMIT:
            return "the problem needs more scratch than apd_attn_paged_decode_noalloc's built-in "
                   "APD_NOALLOC_SCRATCH_BYTES (use apd_attn_paged_decode with a workspace, or fewer splits)";
        default: return "unknown status";
    }
}

const char* apd_last_cuda_error(void) { return g_last_cuda_error; }

}  // extern "C"

int apd_selftest_shared_ring_release(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                                     const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* out,
                                     float scale, void* workspace, size_t workspace_bytes,
                                     uint64_t short_timeout_ns, apd_stream_t stream) {
    if (!page_table) return APD_ERR_NULL_POINTER;
    if (short_timeout_ns == 0 || short_timeout_ns > 1000000000ull) return APD_ERR_ARGUMENT;
    SplitTestHooks h;
    h.wait_ns = short_timeout_ns;
    h.skip_release = 1;
    return decode_impl(q, k_cache, v_cache, page_table, seq_lens, out, scale, 0, workspace, workspace_bytes, stream,
                       nullptr, &h);
}

int apd_selftest_mq_tc_stall(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                             const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* out,
                             float scale, int num_splits, void* workspace, size_t workspace_bytes,
                             uint64_t short_timeout_ns, apd_stream_t stream) {
    if (!page_table) return APD_ERR_NULL_POINTER;
    if (short_timeout_ns == 0 || short_timeout_ns > 1000000000ull) return APD_ERR_ARGUMENT;
    SplitTestHooks h;
    h.wait_ns = short_timeout_ns;
    h.skip_pfull = 1;
    return decode_impl(q, k_cache, v_cache, page_table, seq_lens, out, scale, num_splits, workspace, workspace_bytes,
                       stream, nullptr, &h);
}

int apd_selftest_bounded_wait(uint32_t* out, uint64_t short_timeout_ns, apd_stream_t stream) {
    if (!out) return APD_ERR_NULL_POINTER;
    if (short_timeout_ns == 0 || short_timeout_ns > 1000000000ull) return APD_ERR_ARGUMENT;
    cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(out, 0, 4 * sizeof(uint32_t), st);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(selftest)");
    apd::wait_selftest_kernel<<<1, 64, 0, st>>>(out, short_timeout_ns);
    e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, "wait_selftest_kernel launch");
    return APD_OK;
}
