/*
 * attn_paged_decode.h -- C ABI of the B200 (sm_100a) paged split-KV decode
 * attention library (libattn_paged_decode.so).
 *
 * Operation (AstrAI commit d565d44c, csrc/kernels/attn_paged_decode.cu, commit
 * log: the attn_paged_decode entry, its scalar and MMA split-KV decode kernels,
 * the o_part / ml_part partials and the single combine kernel):
 *
 *   single-token decode attention over a paged bf16 KV cache.  For every
 *   sequence b and query head h, with g = Hq / Hkv, kv head kvh = h / g and
 *   L = seq_lens[b]:
 *       s_t   = scale * <q[b,h,:], K_t>          for t in [0, L)
 *       out[b,h,:] = sum_t softmax(s)_t * V_t    (L == 0 -> zeros)
 *   where K_t / V_t are row (page_table[b][t / P], t % P, kvh, :) of
 *   k_cache / v_cache.  Decode is causal, so the one query token sees all L
 *   stored positions.  The KV range of each (sequence, kv head) is split across
 *   workers (split-KV); each split leaves a partial output with its running max
 *   and sum, and one combine kernel merges them.  Query heads that share a kv
 *   head are processed together, so K/V leave HBM once per kv head (above 64
 *   query heads per kv head at head_dim 128, blocks of at most 64 of them read
 *   the same tiles at about the same time, the repeats from L2).
 *
 * Ownership and threading.  The caller owns every buffer, including the
 * workspace.  The library allocates nothing, never synchronises the stream and
 * never reads device memory on the host, so a call can be captured in a CUDA
 * graph once the workspace exists.  Work is enqueued on `stream` in stream
 * order; a call returns as soon as the kernels are launched.  Calls may be made
 * from several host threads; calls that share a workspace must be ordered on
 * the device (same stream, or events).
 *
 * Errors.  Every entry point returns an apd_status.  Argument faults are found
 * on the host before anything is launched; nothing is written then.  A failed
 * CUDA launch returns APD_ERR_CUDA.  Device-side contract violations (see
 * apd_attn_paged_decode) never fault: they are clamped or read as zeros and
 * recorded as sticky bits in the workspace, which apd_read_device_flags reads.
 * No C++ exception crosses this interface.
 */
#ifndef ATTN_PAGED_DECODE_H_
#define ATTN_PAGED_DECODE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define APD_VERSION 1

/* A CUDA stream handle; identical to cudaStream_t (NULL = legacy default stream). */
typedef struct CUstream_st* apd_stream_t;

typedef enum apd_dtype {
    APD_DTYPE_BF16 = 1,
    APD_DTYPE_INT32 = 2,
    APD_DTYPE_FP32 = 3,
    APD_DTYPE_UINT8 = 4
} apd_dtype;

/* A strided view of device memory.  `stride` is in elements; only the first
 * `ndim` entries of shape/stride are read.  Dimensions of extent 1 may carry
 * any stride. */
typedef struct apd_tensor {
    void* data;
    int32_t dtype;     /* apd_dtype */
    int32_t ndim;
    int64_t shape[4];
    int64_t stride[4];
} apd_tensor;

typedef enum apd_status {
    APD_OK = 0,
    APD_ERR_NULL_POINTER = 1,     /* a descriptor or its data pointer is NULL            */
    APD_ERR_DTYPE = 2,            /* q/k/v/out not bf16, page_table/seq_lens not int32    */
    APD_ERR_SHAPE = 3,            /* ndim or extents disagree between the tensors         */
    APD_ERR_GQA = 4,              /* num_q_heads is not a multiple of num_kv_heads        */
    APD_ERR_HEAD_DIM = 5,         /* head_dim not in {32, 64, 128, 256}                   */
    APD_ERR_LAYOUT = 6,           /* head dim not contiguous, or a stride / base pointer
                                     not 16-byte aligned                                  */
    APD_ERR_PAGE_SIZE = 7,        /* page_size not a positive multiple of 32              */
    APD_ERR_NUM_SPLITS = 8,       /* num_splits < 0                                       */
    APD_ERR_WORKSPACE = 9,        /* workspace NULL, not 256-byte aligned, or too small   */
    APD_ERR_TOO_LARGE = 10,       /* batch > APD_MAX_BATCH or indices would overflow      */
    APD_ERR_CUDA = 11,            /* a CUDA runtime call or a kernel launch failed        */
    APD_ERR_ARGUMENT = 12,        /* any other bad argument (e.g. a NULL output pointer)  */
    APD_ERR_SCRATCH_LIMIT = 13    /* apd_attn_paged_decode_noalloc: the problem needs more
                                     scratch than APD_NOALLOC_SCRATCH_BYTES               */
} apd_status;

/* Largest batch one call accepts (the per-sequence lengths and their prefix
 * sums are staged in shared memory). */
#define APD_MAX_BATCH 4096

/* Sticky device flags (apd_read_device_flags). */
#define APD_FLAG_PAGE_OUT_OF_RANGE 0x1u /* a page-table entry outside [0, num_pages): read as zeros */
#define APD_FLAG_SEQ_LEN_CLAMPED   0x2u /* seq_len > max_pages_per_seq * page_size: clamped         */
#define APD_FLAG_SEQ_LEN_NEGATIVE  0x4u /* seq_len < 0: treated as 0                                */
#define APD_FLAG_WAIT_TIMEOUT      0x8u /* an async copy did not complete in time: output invalid  */

/*
 * apd_workspace_size -- bytes of device workspace that apd_attn_paged_decode
 * needs for this problem shape (workspace pattern of the AstrAI commit log:
 * the decode partials are preallocated once and reused by every call, which is
 * what makes the call capturable in a CUDA graph).
 *
 *   batch, num_q_heads, num_kv_heads, head_dim: as in apd_attn_paged_decode.
 *   num_splits: the value that will be passed to apd_attn_paged_decode.
 *     num_splits >= 1 needs room for batch * num_kv_heads * ceil(g/16) *
 *     num_splits partial slots; num_splits == 0 ("auto") needs room for two
 *     slots per hardware worker of the current CUDA device (148 SMs are assumed
 *     when no device is visible).  A smaller auto workspace still works: the
 *     call then uses fewer parallel workers.
 *
 * Returns 0 if the arguments are invalid.  Does not allocate.  The returned
 * size is a multiple of 256; the workspace must be 256-byte aligned.
 */
size_t apd_workspace_size(int batch, int num_q_heads, int num_kv_heads, int head_dim, int num_splits);

/*
 * apd_workspace_init -- zero a workspace (all workspace_bytes of it), enqueued on
 * `stream`, which clears the sticky device flags.  Optional: correct output does
 * not depend on the workspace's contents.
 */
int apd_workspace_init(void* workspace, size_t workspace_bytes, apd_stream_t stream);

/*
 * apd_attn_paged_decode -- the decode attention call.
 *
 *   q          bf16 [B, Hq, D], stride(D) == 1, other strides multiples of 8
 *              elements, base 16-byte aligned.
 *   k_cache    bf16 [num_pages, page_size, Hkv, D] (logical "NHD" order); any
 *   v_cache    strides that keep D contiguous and are multiples of 8 elements,
 *              so "HND" storage [num_pages, Hkv, page_size, D] is passed as the
 *              permuted view.  k_cache and v_cache have the same shape.
 *   page_table int32 [B, max_pages_per_seq]; entry [b][j] is the physical page
 *              holding tokens [j*P, (j+1)*P) of sequence b.  Entries at or past
 *              ceil(seq_lens[b] / P) are never read.
 *   seq_lens   int32 [B], on the device; read only by the kernels.
 *   out        bf16 [B, Hq, D], stride(D) == 1, written for every (b, h).
 *   scale      multiplies the q.K dot products (typically 1/sqrt(D)).
 *   num_splits 0 = auto: the KV work of all sequences and kv heads is cut into
 *              equal runs of 32-token tiles, one run per hardware worker, so
 *              every SM gets the same number of tiles and longer sequences get
 *              more splits (the ejkernel PageAttentionConfig convention that
 *              num_splits = 0 means automatic).
 *              k >= 1: sequence b is split into min(k, n_b) page-aligned chunks
 *              of ceil(n_b / min(k, n_b)) 32-token tiles, n_b = ceil(L_b / 32);
 *              k == 1 means no split-KV and a single kernel launch.
 *   workspace  device memory of at least apd_workspace_size(...) bytes, 256-byte
 *              aligned, owned by the caller; its contents between calls are
 *              scratch except for the sticky flags word.
 *   stream     CUDA stream the kernels are enqueued on.
 *
 * Requirements checked on the host (status codes above): Hq % Hkv == 0,
 * D in {32, 64, 128, 256}, page_size % 32 == 0, 0 <= num_splits, B <= APD_MAX_BATCH,
 * alignment of the strided layouts, workspace size.
 *
 * Device-side contract (not checked on the host, since seq_lens and page_table
 * live on the device): 0 <= seq_lens[b] <= max_pages_per_seq * page_size and
 * the first ceil(seq_lens[b] / page_size) page-table entries of sequence b lie in
 * [0, num_pages).  Violations never fault: lengths are clamped, pages outside
 * the pool read as zeros, and the matching APD_FLAG_* bit is set.
 *
 * Numerics: bf16 inputs, fp32 accumulation (tensor cores), softmax in fp32
 * with exp2, probabilities rounded to bf16 for the PV product, output rounded
 * to bf16 (nearest-even).  Results are deterministic for a given device, shape
 * and num_splits.
 */
int apd_attn_paged_decode(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                          const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* out,
                          float scale, int num_splits, void* workspace, size_t workspace_bytes,
                          apd_stream_t stream);

/*
 * apd_attn_paged_decode_ex -- apd_attn_paged_decode with launch options.
 *
 * Same arguments, checks, results and errors as apd_attn_paged_decode, plus
 * `options` (may be NULL, which makes the two calls identical):
 *   split_done_event  a cudaEvent_t (created by the caller) that is recorded on
 *                     `stream` right after the split kernel is enqueued, before
 *                     the combine kernel; lets a caller time the split kernel
 *                     alone with events.  Recording it between the kernels
 *                     also turns off the programmatic (PDL) overlap of the
 *                     combine kernel's launch for that call.  While `stream`
 *                     is being captured into a CUDA graph the event is recorded
 *                     as an external event-record node, so it also times the
 *                     kernel in every replay of the graph.
 *   disable_pdl       nonzero: launch the combine kernel without programmatic
 *                     dependent launch.
 *   host_seq_lens     NULL, or host memory holding the B sequence lengths as the
 *                     caller knows them on the host (the values seq_lens holds on
 *                     the device).  A planning hint for num_splits == 0, read during
 *                     the call (and baked into a CUDA graph captured around it):
 *                     when every (sequence, kv head, head block) unit can have a CTA
 *                     of its own on a distinct SM and the longest unit is no longer
 *                     than the balanced plan's share per CTA (within 3% plus about
 *                     the combine kernel's cost), the call runs one kernel whose
 *                     CTAs each own one unit and merge its parts in shared memory
 *                     (plan mode 2), with no partials and no combine kernel.
 *                     Otherwise the plan is the one without the hint.  The kernels
 *                     always read the lengths from the device seq_lens, so a hint
 *                     that differs from them changes the speed, never the result
 *                     beyond rounding.  Mode 2 is the one plan that is not bitwise
 *                     reproducible: its warps take the unit's tiles in the order
 *                     they become free (the fastest order measured), so the parts
 *                     they merge, and the last bits of the output, can differ from
 *                     call to call (always within the accuracy of the other plans).
 *                     Without the hint, and with fixed splits, every call on the
 *                     same inputs gives the same bits.
 */
typedef struct apd_launch_options {
    void* split_done_event;       /* cudaEvent_t or NULL */
    int32_t disable_pdl;
    int32_t reserved;             /* must be 0 */
    const int32_t* host_seq_lens; /* NULL or int32[B] in host memory */
} apd_launch_options;

int apd_attn_paged_decode_ex(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                             const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* out,
                             float scale, int num_splits, void* workspace, size_t workspace_bytes,
                             apd_stream_t stream, const apd_launch_options* options);

/*
 * apd_attn_contig_decode -- the same decode attention over a contiguous (not
 * paged) KV cache: the ContigKV addressing policy next to PagedKV in the AstrAI
 * commit log of csrc/kernels/attn_paged_decode.cu (attn_kv_source.cuh with
 * ContigKV/PagedKV, kernels templated on the KV policy, stride-based addressing
 * for the "bhld" / "blhd" layouts).
 *
 *   k, v       bf16 [B, Lmax, Hkv, D] in logical "blhd" order, D contiguous, other
 *              strides multiples of 8 elements: "bhld" storage [B, Hkv, Lmax, D] is
 *              passed as the permuted view.  Lmax is any positive length (not
 *              necessarily a multiple of 32).  Token t of sequence b is
 *              k[b, t, kvh, :].
 *   q, seq_lens, out, scale, num_splits, workspace, stream: as in
 *              apd_attn_paged_decode (same workspace size).  Device contract:
 *              0 <= seq_lens[b] <= Lmax (larger values are clamped and flagged).
 *
 * It runs the paged kernels with one Lmax-token page per sequence (page b), so a
 * paged and a contiguous cache holding the same tokens give identical results.
 */
int apd_attn_contig_decode(const apd_tensor* q, const apd_tensor* k, const apd_tensor* v, const apd_tensor* seq_lens,
                           const apd_tensor* out, float scale, int num_splits, void* workspace,
                           size_t workspace_bytes, apd_stream_t stream);

/* apd_attn_contig_decode with launch options (see apd_attn_paged_decode_ex). */
int apd_attn_contig_decode_ex(const apd_tensor* q, const apd_tensor* k, const apd_tensor* v,
                              const apd_tensor* seq_lens, const apd_tensor* out, float scale, int num_splits,
                              void* workspace, size_t workspace_bytes, apd_stream_t stream,
                              const apd_launch_options* options);

/*
 * apd_attn_paged_prefill -- multi-query (chunked prefill) attention over the same
 * paged cache (AstrAI commit log of csrc/kernels/attn_paged_decode.cu: prefill
 * kernels templated on the paged KV policy, the unified causal_offset, and 2-D /
 * 3-D masks that may be combined with causal).
 *
 *   q          bf16 [B, Lq, Hq, D] (Lq >= 1 new query tokens per sequence), D
 *              contiguous, other strides multiples of 8 elements, base 16-byte
 *              aligned.
 *   k_cache, v_cache, page_table, seq_lens, scale: as in apd_attn_paged_decode;
 *              seq_lens[b] keys are stored for sequence b.
 *   mask       NULL, or uint8 [B, kv_len] (one row per sequence) or [B, Lq, kv_len]
 *              (one row per query), nonzero = visible, kv_len >=
 *              max_pages_per_seq * page_size, any non-negative strides.
 *   out        bf16 [B, Lq, Hq, D], same layout rules as q.
 *   causal_offset  -1: no causal mask; c >= 0: query i sits at position c + i and
 *              sees keys t <= c + i.
 *
 * Query i of sequence b sees key t when t < seq_lens[b], the causal rule allows it
 * and the mask (if any) is nonzero at t; the output is the softmax-weighted sum of
 * the visible V rows, or zeros when no key is visible.  One kernel launch, no
 * workspace, no split of the key range (each CTA streams its rows' whole range).
 * Same threading, error and device-contract conventions as apd_attn_paged_decode.
 */
int apd_attn_paged_prefill(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                           const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* mask,
                           const apd_tensor* out, float scale, int causal_offset, apd_stream_t stream);

/*
 * apd_attn_paged_prefill_ex -- apd_attn_paged_prefill with the kernel chosen by
 * the caller (same result within the tolerance; for A/B measurement and tests).
 *
 *   kernel  APD_PREFILL_AUTO (0): what apd_attn_paged_prefill uses;
 *           APD_PREFILL_MMA_SYNC (1): warp-level mma.sync tiles, every head dim;
 *           APD_PREFILL_TCGEN05 (2): fifth-generation tensor cores (tcgen05.mma
 *           with TMEM accumulators, 128 query rows x 128 keys per step, 64 keys
 *           for D = 256); every head dim.
 *   Any other value -> APD_ERR_ARGUMENT, before any launch.
 */
#define APD_PREFILL_AUTO 0
#define APD_PREFILL_MMA_SYNC 1
#define APD_PREFILL_TCGEN05 2
int apd_attn_paged_prefill_ex(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                              const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* mask,
                              const apd_tensor* out, float scale, int causal_offset, apd_stream_t stream,
                              int kernel);

/*
 * apd_attn_paged_decode_noalloc -- the same decode call for callers that cannot
 * allocate device memory.  The pages have no counterpart of this entry point.
 *
 * Some callers have no way to obtain a workspace: a plugin handed only its input
 * and output tensors by a host framework that owns every device allocation; code
 * that runs under a fixed device-memory budget where a side allocation is not
 * allowed; or code on a latency path where cudaMalloc, which can synchronise the
 * device, is not acceptable.  This entry point needs no workspace: its scratch
 * (the split partials, their running max and sum, and the per-sequence tile
 * prefix sums) lives in one file-scope static device array of
 * APD_NOALLOC_SCRATCH_BYTES, which every GPU that loads the library holds until
 * the process exits.  It calls no cudaMalloc, cudaFree or other allocating
 * routine.
 *
 *   Arguments, layouts, checks, numerics and errors are those of
 *   apd_attn_paged_decode, without `workspace` / `workspace_bytes`.
 *   num_splits 0 (auto) plans as many parallel workers as the scratch holds
 *              partials for (all of them for common shapes); num_splits >= 1
 *              needs apd_workspace_size(...) <= APD_NOALLOC_SCRATCH_BYTES.
 *   Returns APD_ERR_SCRATCH_LIMIT, before anything is launched, when the
 *   problem needs more scratch than the array holds.
 *
 * Set-up: the first call on each device (with that device current) looks up the
 * array's device address with cudaGetSymbolAddress, which can load the library's
 * device code; make that first call before any stream capture.
 *
 * Sharing: every call in the process uses the same array on a given device, and
 * the array keeps whatever the last call left in it.  No part of it has to start
 * at zero (each call writes every partial and prefix sum it later reads).  Calls
 * that can overlap on the GPU (unordered streams) race on the array and may
 * return wrong results; order them on one stream or with events.  The sticky
 * device flags of this entry point go to the array and are not reported.
 */
#define APD_NOALLOC_SCRATCH_BYTES (8u << 20) /* 8 MiB per device */

int apd_attn_paged_decode_noalloc(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                                  const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* out,
                                  float scale, int num_splits, apd_stream_t stream);

/*
 * apd_gemv_bf16 -- the decode projection y = x W^T of a bf16 linear layer with a
 * few activation rows (AstrAI commit logs of astrai/extension/ops/gemv.py and
 * docs/developer/decode_linear_benchmark.md: the bf16 GEMV that decode-time
 * linear layers use for M = 1..8, weights [out_features, in_features]).
 *
 *   x          bf16 [M, K], 1 <= M <= APD_GEMV_MAX_M, K a multiple of 8, K
 *              contiguous, row stride a multiple of 8 elements, base 16-byte
 *              aligned.
 *   w          bf16 [N, K] with the same layout rules (a linear layer's weight).
 *   y          bf16 [M, N], any strides (2-byte aligned); y[m][n] =
 *              sum_k x[m][k] * w[n][k], accumulated in fp32 on tensor cores and
 *              rounded to bf16 (nearest-even).
 *   workspace  at least apd_gemv_workspace_size(M, N, K) bytes, 256-byte aligned,
 *              caller-owned; scratch between calls (calls sharing a workspace must
 *              be ordered on the device).
 *
 * Same conventions as apd_attn_paged_decode: no allocation, no synchronisation,
 * stream-ordered, capturable in a CUDA graph; argument faults are returned
 * before anything is launched.
 */
#define APD_GEMV_MAX_M 8

size_t apd_gemv_workspace_size(int m, int n, int k);

int apd_gemv_bf16(const apd_tensor* x, const apd_tensor* w, const apd_tensor* y, void* workspace,
                  size_t workspace_bytes, apd_stream_t stream);

/*
 * apd_gemv_query_plan -- how apd_gemv_bf16 launches an [M, K] x [N, K]^T product:
 * the weight matrix is cut into units of 16 rows x 256 columns that `workers` warps
 * share equally (or, with one to four 16-row tiles per SM and rows of at most 2048
 * columns, each warp takes whole 16-row tiles; or, for weights of at most 32 MB with
 * fewer 16-row tiles than SMs, each CTA takes one tile and splits its columns).  sm_count > 0 plans for a device with
 * that many SMs without touching CUDA; sm_count <= 0 queries the current device.
 * Returns APD_ERR_ARGUMENT for M outside 1..APD_GEMV_MAX_M or N, K < 1.
 */
typedef struct apd_gemv_plan {
    int32_t workers;        /* warps sharing the weight stream                          */
    int32_t grid_ctas;      /* CTAs of the GEMV kernel                                  */
    int32_t warps_per_cta;
    int32_t stages;         /* async-copy ring depth per warp                           */
    int32_t x_staged;       /* 1: x is copied once per CTA into shared memory            */
    int32_t sum_ctas;       /* CTAs of the partial-sum kernel; 0 when it is not launched */
    int32_t cta_per_mtile;  /* 1: CTA b owns 16-row tile b; its warps split K and add their
                               parts in shared memory (one kernel, no partials)        */
    int64_t workspace_bytes;
} apd_gemv_plan;

int apd_gemv_query_plan(int m, int n, int k, int sm_count, apd_gemv_plan* plan);

/*
 * apd_read_device_flags -- synchronise `stream`, copy the sticky APD_FLAG_* word
 * out of the workspace into *flags and, if `clear` is nonzero, reset it.  A
 * debugging / testing aid: it blocks the host, so it does not belong in a
 * captured or latency-critical loop.
 */
int apd_read_device_flags(const void* workspace, size_t workspace_bytes, apd_stream_t stream, uint32_t* flags,
                          int clear);

/*
 * apd_selftest_bounded_wait -- exercises, on the GPU, the bounded waits every kernel
 * here uses on its mbarriers, without any copy, MMA or fault: one thread waits on an
 * mbarrier that nothing completes, with a limit of `short_timeout_ns` (1 .. 1e9 ns),
 * and must give up, set APD_FLAG_WAIT_TIMEOUT and raise the CTA's abort flag; a second
 * thread waits on another such mbarrier with the kernels' full limit (2 s) and must give
 * up early because of that abort flag.
 *
 *   out      device uint32[4] (caller-owned): out[0] = 1 if the first wait gave up,
 *            out[1] = 1 if the second gave up, out[2] = the second wait's duration in
 *            microseconds, out[3] = the flag word written by the first wait.
 *   Returns APD_ERR_NULL_POINTER / APD_ERR_ARGUMENT before any launch, APD_ERR_CUDA on a
 *   launch failure, else APD_OK (asynchronous: read `out` after synchronising `stream`).
 */
int apd_selftest_bounded_wait(uint32_t* out, uint64_t short_timeout_ns, apd_stream_t stream);

/*
 * apd_selftest_shared_ring_release -- exercises, on the GPU and without any fault, the
 * error path of the shared K/V ring (auto splits with more than 16 query heads per kv
 * head, where the head blocks of a kv head share one ring that the first of them fills
 * and the others release stage by stage).  It runs apd_attn_paged_decode(num_splits = 0)
 * on the given problem with two differences: the followers never release a stage, and
 * every mbarrier wait gives up after `short_timeout_ns` (1 .. 1e9 ns) instead of 2 s.
 * Each ring's leader must then give up on its first refill, stop issuing copies, wait
 * (bounded) for its copies in flight and return; its followers must give up on their
 * next wait through the CTA's abort word.  The call ends within a few limits, the flag
 * word in the workspace gets APD_FLAG_WAIT_TIMEOUT, and `out` is undefined.
 *
 *   Arguments as apd_attn_paged_decode with num_splits = 0.  Returns APD_ERR_ARGUMENT
 *   before any launch when the problem does not take the shared ring (16 or fewer q
 *   heads per kv head) or the limit is out of range; otherwise as that call.
 */
int apd_selftest_shared_ring_release(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                                     const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* out,
                                     float scale, void* workspace, size_t workspace_bytes,
                                     uint64_t short_timeout_ns, apd_stream_t stream);

/*
 * apd_selftest_mq_tc_stall -- exercises, on the GPU and without any fault, the error path
 * of the tensor-core multi-query kernel (apd_plan.mode 3: more than 16 q heads per kv head
 * at head_dim 128).  It runs apd_attn_paged_decode(num_splits) on the given problem with two
 * differences: the softmax warps never hand over the weights P of their second tile, and
 * every wait gives up after `short_timeout_ns` (1 .. 1e9 ns) instead of 2 s.  The MMA
 * issuer and the softmax warps must then give up, raise the CTA's abort flag, leave their
 * loops together (the softmax warps through a barrier vote), wait (bounded) for their
 * copies and MMAs in flight and meet before the TMEM columns are freed and, with the
 * cluster merge, at the cluster barrier.  The call ends within a few limits, the flag word
 * in the workspace gets APD_FLAG_WAIT_TIMEOUT, and `out` is undefined.
 *
 *   Arguments as apd_attn_paged_decode.  Returns APD_ERR_ARGUMENT before any launch when
 *   the problem does not take the tensor-core kernel or the limit is out of range;
 *   otherwise as that call.
 */
int apd_selftest_mq_tc_stall(const apd_tensor* q, const apd_tensor* k_cache, const apd_tensor* v_cache,
                             const apd_tensor* page_table, const apd_tensor* seq_lens, const apd_tensor* out,
                             float scale, int num_splits, void* workspace, size_t workspace_bytes,
                             uint64_t short_timeout_ns, apd_stream_t stream);

/* apd_plan -- how a call with these arguments would be launched (for tests,
 * benchmarks and profiling). */
typedef struct apd_plan {
    int32_t mode;              /* 0 = balanced (num_splits == 0), 1 = fixed splits,
                                  2 = one CTA per unit, parts merged in shared memory
                                  (num_splits == 0 with host lengths, see
                                  apd_launch_options.host_seq_lens),
                                  3 = tensor-core multi-query kernel (more than
                                  16 q heads per kv head at head_dim 128, any
                                  num_splits): one CTA per split of each
                                  (sequence, kv head, q-head block)             */
    int32_t num_workers;       /* warps that each own a run of tiles             */
    int32_t grid_ctas;         /* CTAs of the split kernel                       */
    int32_t warps_per_cta;
    int32_t stages;            /* async-copy ring depth per warp (per kv head
                                  when shared_kv_ring = 1)                      */
    int32_t rows_per_unit;     /* query heads packed per unit (<= 16)            */
    int32_t head_blocks;       /* ceil(g / 16)                                   */
    int32_t combine_ctas;      /* 0 when no combine kernel is launched           */
    int64_t smem_bytes;        /* dynamic shared memory of the split kernel      */
    int64_t partial_slots;
    int64_t workspace_bytes;   /* bytes the call needs                           */
    int32_t shared_kv_ring;    /* 1: balanced mode with g > 16; the head_blocks
                                  warps of a kv head sit in one CTA and read K/V
                                  from one ring that the first of them fills, so
                                  each K/V tile leaves HBM once (warps_per_cta is
                                  then a multiple of head_blocks)               */
    int32_t cluster_size;      /* mode 3: the splits of a unit run as one thread-block
                                  cluster of this many CTAs and merge in the kernel
                                  (no combine kernel); 0 otherwise               */
    int32_t q_head_blocks;     /* mode 3: CTAs per split of a (sequence, kv head),
                                  each owning one block of its query heads:
                                  ceil(g / 64); 1 otherwise                      */
    int32_t q_heads_per_block; /* mode 3: query heads of a block but the last,
                                  ceil(g / q_head_blocks) rounded up to 16; 0
                                  otherwise                                      */
} apd_plan;

/* apd_query_plan -- fills *plan.  workspace_bytes: the size that will be passed
 * (SIZE_MAX = unlimited).  sm_count > 0 plans for a device with that many SMs
 * without touching CUDA (host-side planning, e.g. for tests); sm_count <= 0
 * queries the current CUDA device. */
int apd_query_plan(int batch, int num_q_heads, int num_kv_heads, int head_dim, int num_splits,
                   size_t workspace_bytes, int sm_count, apd_plan* plan);

/* apd_query_plan_ex -- apd_query_plan for a call given host_seq_lens (int32[batch] in
 * host memory, or NULL) and the longest length the cache holds, max_seq_len =
 * max_pages_per_seq * page_size (Lmax for a contiguous cache); lengths are clamped
 * to [0, max_seq_len] as the kernels clamp them. */
int apd_query_plan_ex(int batch, int num_q_heads, int num_kv_heads, int head_dim, int num_splits,
                      size_t workspace_bytes, int sm_count, const int32_t* host_seq_lens, int64_t max_seq_len,
                      apd_plan* plan);

/* apd_status_string -- human-readable text for an apd_status (never NULL; unknown codes
 * give "unknown status").  The statuses are the argument checks that the AstrAI commit
 * log of csrc/kernels/attn_paged_decode.cu lists for the decode entry (q_head divisible
 * by kv_head, head-dim contiguity, the split-KV scratch and output layout), plus this
 * library's own size, workspace and CUDA failures.  The returned string is static: do
 * not free it. */
const char* apd_status_string(int status);

/* Text of the last CUDA error seen by this thread inside the library ("" if none). */
const char* apd_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* ATTN_PAGED_DECODE_H_ */
