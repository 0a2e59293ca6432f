/*
 * hsa.h -- C ABI of the B200 (sm_100a) hierarchical indexed sparse attention
 * (HISA) library, libhsa.so.
 *
 * The method (page "HISA: Hierarchical Indexed Sparse Attention",
 * discuz.ruhao.net thread 187): a drop-in replacement for the token-level
 * indexer of DeepSeek sparse attention (DSA). For every query position t the
 * causal key prefix is cut into blocks of B tokens (section 第一步); each block
 * gets a representative vector, the blocks are scored with the indexer's own
 * rule and the best m are kept, the first block and the query's own (last)
 * block always among them (the forced first/last block note). Only the
 * tokens inside the kept blocks are then scored and the best k kept
 * (section 第二步); the output has the original indexer's format and the
 * attention that follows is the unchanged sparse softmax attention over those
 * k tokens, shared by all H query heads of a multi-query layer (the
 * "drop-in replacement" paragraph). The indexer cost falls from O(L^2) to
 * O(L^2/B + L*m*B) (the complexity paragraph).
 *
 * Readings fixed by this library where the pages are silent:
 *   - scoring rule: plain dot product q_idx[t] . k_idx[j] (one indexer head);
 *   - block representative: fp32 sum of the block's B key rows;
 *   - the m kept blocks include the two forced ones; the other m-2 are the
 *     best-scoring complete blocks among 1 .. floor(t/B)-1;
 *   - causal keys are j <= t; ties go to the lowest index;
 *   - indices are written ascending and padded with -1;
 *   - softmax scale defaults to 1/sqrt(d).
 *
 * Conventions for every call:
 *   - All tensor pointers are DEVICE pointers to dense row-major arrays owned
 *     by the caller; the library never allocates, frees or synchronises on the
 *     hot path. bf16 tensors are passed as 16-bit bit patterns (hsa_bf16).
 *   - Pointers must be 16-byte aligned and the row lengths below must keep
 *     every row 16-byte aligned (d_idx and d are multiples of 8).
 *   - Work is enqueued on `stream`; the call returns once it is enqueued.
 *   - Every argument is checked on the host before anything is launched; on
 *     a failed check nothing is launched and an HSA_ERR_* code is returned.
 *     No exception crosses this boundary. Non-finite inputs are not checked.
 *   - Indexer inputs holding integer values of magnitude <= 8 (the synthetic
 *     workloads) give exact fp32 scores, so selections are reproducible bit
 *     for bit; for general real inputs near-ties may order differently from a
 *     sequential CPU evaluation.
 */
#ifndef HSA_H_
#define HSA_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define HSA_API __attribute__((visibility("default")))
#else
#define HSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef uint16_t hsa_bf16; /* bf16 bit pattern */

enum {
  HSA_OK = 0,
  HSA_ERR_ARG = 1,       /* null / misaligned pointer or unsupported size  */
  HSA_ERR_WORKSPACE = 2, /* workspace missing or smaller than required      */
  HSA_ERR_CUDA = 3,      /* a CUDA launch or runtime call failed            */
  HSA_ERR_TIMEOUT = 4,   /* a bounded device-side wait gave up (reported by
                            hsa_device_status)                              */
  HSA_ERR_DEVICE = 5     /* current device is not sm_100 (B200 class)       */
};

/* Method and layer sizes. */
typedef struct hsa_params {
  int32_t B;     /* tokens per block, 1 <= B <= 1024                           */
  int32_t m;     /* kept blocks per query incl. the 2 forced ones, 2 <= m <= 512;
                    m*B <= 65536 candidates for B in {64, 128, 256} (scored on
                    tensor cores), m*B <= 16384 for other block sizes         */
  int32_t k;     /* kept tokens per query, 1 <= k <= 8192 (k >= m*B keeps every
                    candidate of the kept blocks)                              */
  int32_t d_idx; /* indexer head dim: 64 or 128                                 */
  int32_t H;     /* query heads sharing one K/V head: 1 <= H <= 128 (one pass of
                    the attention per group of up to 64 heads)                */
  int32_t d;     /* attention head dim: 64 or 128                               */
  float scale;   /* softmax scale; 0 selects 1/sqrt(d)                          */
} hsa_params;

/* Human-readable text for a status code (static storage). */
HSA_API const char* hsa_status_string(int status);

/* Workspace bytes needed by hsa_index / hsa_select_blocks / hsa_select_tokens
 * for Lq queries over Lk keys. Writes *bytes. */
HSA_API int hsa_index_workspace_size(const hsa_params* p, int64_t Lq, int64_t Lk, size_t* bytes);

/* Block representatives (section 第一步).
 *   k_idx [Lk][d_idx] bf16 keys of the indexer.
 *   ksum  [floor(Lk/B)][d_idx] fp32, written: ksum[b][c] = sum_{j in block b} k_idx[j][c].
 * Only complete blocks are produced. */
HSA_API int hsa_block_sums(const hsa_params* p, int64_t Lk, const hsa_bf16* k_idx, float* ksum,
                   cudaStream_t stream);

/* Block-level selection (section 第一步 + forced first/last block).
 * Query i (0 <= i < Lq) sits at absolute position t = Lk - Lq + i.
 *   q_idx  [Lq][d_idx] bf16 indexer queries.
 *   ksum   [floor(Lk/B)][d_idx] fp32 from hsa_block_sums.
 *   blocks [Lq][m] int32, written: kept block ids ascending, -1 padded.
 * With nb = floor(t/B)+1 causal blocks: nb <= m keeps them all; otherwise
 * blocks 0 and nb-1 plus the m-2 best of 1..nb-2 by (score desc, id asc). */
HSA_API int hsa_select_blocks(const hsa_params* p, int64_t Lq, int64_t Lk, const hsa_bf16* q_idx,
                      const float* ksum, int32_t* blocks, void* workspace,
                      size_t workspace_bytes, cudaStream_t stream);

/* Token-level selection inside the kept blocks (section 第二步).
 *   q_idx [Lq][d_idx], k_idx [Lk][d_idx] bf16; blocks [Lq][m] from hsa_select_blocks.
 *   indices [Lq][k] int32, written ascending, -1 padded.
 * Candidates are the tokens j <= t of the kept blocks; if there are at most k
 * of them all are kept, else the k best by (score desc, j asc). */
HSA_API int hsa_select_tokens(const hsa_params* p, int64_t Lq, int64_t Lk, const hsa_bf16* q_idx,
                      const hsa_bf16* k_idx, const int32_t* blocks, int32_t* indices,
                      void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* The whole indexer: block sums, block selection and token selection.
 *   q_idx [Lq][d_idx], k_idx [Lk][d_idx] bf16 -> indices [Lq][k] int32.
 * Requires 1 <= Lq <= Lk and Lk/B <= 16384 blocks. workspace:
 * hsa_index_workspace_size bytes. */
HSA_API int hsa_index(const hsa_params* p, int64_t Lq, int64_t Lk, const hsa_bf16* q_idx,
              const hsa_bf16* k_idx, int32_t* indices, void* workspace, size_t workspace_bytes,
              cudaStream_t stream);

/* Sparse softmax attention over the kept tokens (the unchanged downstream
 * attention of the "drop-in replacement" paragraph; softmax(q K^T * scale) V
 * as in the HiLS page's Step 4), multi-query: all H heads share the indices.
 *   Q [Lq][H][d] bf16; K, V [Lk][d] bf16; indices [Lq][k] int32 (entries < 0
 *   are skipped, entries must be < Lk); O [Lq][H][d] bf16, written.
 * fp32 accumulation, O rounded once to bf16. A row without any valid index
 * yields zeros. Two kernel launches per group of 64 heads: the second takes
 * again the rows whose weights outgrew the first's running maxima; the rows
 * it takes are listed in one of 64 device-side slots, taken in turn by the
 * calls (and head groups) of the process, so at most 64 head groups may be
 * in flight at once across streams (a captured CUDA graph keeps the slot of
 * its capture). */
HSA_API int hsa_sparse_attn(const hsa_params* p, int64_t Lq, int64_t Lk, const hsa_bf16* Q,
                    const hsa_bf16* K, const hsa_bf16* V, const int32_t* indices, hsa_bf16* O,
                    cudaStream_t stream);

/* Device workspace bytes for hsa_prefill_host: device copies of its inputs
 * and outputs plus the indexer's workspace. Checks the arguments as
 * hsa_index and hsa_sparse_attn do (no device needed). Writes *bytes. */
HSA_API int hsa_prefill_host_workspace_size(const hsa_params* p, int64_t Lq, int64_t Lk, size_t* bytes);

/* hsa_index followed by hsa_sparse_attn for inputs and outputs in HOST
 * memory: the end-to-end form of the path for a caller whose tensors are not
 * on the device.
 *   q_idx_h [Lq][d_idx], k_idx_h [Lk][d_idx], Q_h [Lq][H][d], K_h/V_h [Lk][d]:
 *     host bf16, read;
 *   O_h [Lq][H][d]: host bf16, written; indices_h [Lq][k]: host int32, written
 *     unless NULL;
 *   workspace: DEVICE memory, 256-byte aligned, of
 *     hsa_prefill_host_workspace_size bytes.
 * Results equal those of hsa_index + hsa_sparse_attn on the same inputs. The
 * queries are cut into at most 16 chunks of whole 128-query tiles. Two copy
 * streams of the library (created on a device's first call, which must not
 * be made during stream capture, and kept until the process exits) fork from
 * `stream` and join back into it: the indexer runs on `stream` while the Q
 * rows come in, the indices go back as soon as the indexer is done, the
 * attention of a chunk starts once its Q rows have landed, and a chunk's O
 * rows go back while the next chunk is computed.
 * All of it is ordered after earlier work on `stream`, and later work on
 * `stream` runs after the last copy; the call returns once everything is
 * enqueued (synchronise `stream` before reading O_h). The copies overlap the
 * kernels only when the host buffers are page-locked (cudaHostAlloc,
 * cudaHostRegister); with pageable buffers the results are the same. Calls
 * on one device enqueue one at a time and their copies share the library's
 * streams, in call order. Errors: those of hsa_index and hsa_sparse_attn;
 * argument errors are returned before anything is enqueued; after a failure
 * during enqueueing, `stream` still waits for every copy already enqueued. */
HSA_API int hsa_prefill_host(const hsa_params* p, int64_t Lq, int64_t Lk, const hsa_bf16* q_idx_h,
                             const hsa_bf16* k_idx_h, const hsa_bf16* Q_h, const hsa_bf16* K_h,
                             const hsa_bf16* V_h, hsa_bf16* O_h, int32_t* indices_h,
                             void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Workspace bytes for hsa_decode_step. */
HSA_API int hsa_decode_workspace_size(const hsa_params* p, int32_t batch, int64_t capacity,
                              size_t* bytes);

/* One decode step for `batch` independent sequences (the decode regime the
 * pages describe as one query per step over a growing KV cache).
 * Caches (device, caller-owned, `capacity` rows per sequence, capacity a
 * multiple of B):
 *   k_idx_cache [batch][capacity][d_idx] bf16, K_cache/V_cache [batch][capacity][d] bf16,
 *   ksum_cache  [batch][capacity/B][d_idx] fp32 (block sums of complete blocks;
 *               fill it for the prompt with hsa_block_sums),
 *   ctx_len     [batch] int32: cached tokens per sequence.
 * New token per sequence: q_idx_new/k_idx_new [batch][d_idx], Q_new [batch][H][d],
 *   K_new/V_new [batch][d] (all bf16).
 * The step appends the new token at position t = ctx_len[b], writes the
 * block sum of a block the token completes, selects blocks and tokens for
 * the query at t (keys j <= t), attends, writes O [batch][H][d] bf16 and,
 * if indices_out is not NULL, the kept indices [batch][k]; then ctx_len[b]
 * += 1. A sequence with ctx_len[b] >= capacity is left untouched and its O
 * row is zero. The step's kernels are programmatic dependent launches: each
 * may begin launching while the previous one runs and waits for it before
 * touching memory, so ordering against earlier work on the stream is the
 * usual stream order. */
HSA_API int hsa_decode_step(const hsa_params* p, int32_t batch, int64_t capacity, int32_t* ctx_len,
                    hsa_bf16* k_idx_cache, hsa_bf16* K_cache, hsa_bf16* V_cache,
                    float* ksum_cache, const hsa_bf16* q_idx_new, const hsa_bf16* k_idx_new,
                    const hsa_bf16* Q_new, const hsa_bf16* K_new, const hsa_bf16* V_new,
                    hsa_bf16* O, int32_t* indices_out, void* workspace, size_t workspace_bytes,
                    cudaStream_t stream);

/* Bytes of the library's static scratch array used by
 * hsa_decode_step_noalloc (one array per GPU, held from module load until
 * the process exits). */
#define HSA_NOALLOC_SCRATCH_BYTES (8u << 20)

/* hsa_decode_step without a workspace argument, for callers that cannot
 * allocate device memory at the point where they decode: code running inside
 * a framework that owns every allocation (a plugin's enqueue, an embedded
 * runtime), or a latency-critical serving loop that may not call cudaMalloc
 * after start-up. The pages describe no such interface; it exists only for
 * these callers.
 * Arguments, caches, results and errors are those of hsa_decode_step. The
 * scratch that hsa_decode_step takes as `workspace` lives instead in a
 * static device array of HSA_NOALLOC_SCRATCH_BYTES inside the library; a
 * step needing more (hsa_decode_workspace_size) returns HSA_ERR_WORKSPACE
 * and launches nothing. Nothing is allocated or freed by this call.
 * The first call on a device looks up that device's copy of the array
 * (cudaGetSymbolAddress, with that device current); make that first call
 * before capturing the stream into a CUDA graph. Every call on a device
 * shares the one array and leaves its contents behind: two calls whose work
 * overlaps on the GPU (different streams without ordering) race on it.
 * The looked-up address is kept for the life of the process: after
 * cudaDeviceReset on a device, the library's per-device state for that device
 * (this address, and the copy streams of hsa_prefill_host) is stale, so do not
 * call into the library on a device that has been reset. */
HSA_API int hsa_decode_step_noalloc(const hsa_params* p, int32_t batch, int64_t capacity,
                                    int32_t* ctx_len, hsa_bf16* k_idx_cache, hsa_bf16* K_cache,
                                    hsa_bf16* V_cache, float* ksum_cache,
                                    const hsa_bf16* q_idx_new, const hsa_bf16* k_idx_new,
                                    const hsa_bf16* Q_new, const hsa_bf16* K_new,
                                    const hsa_bf16* V_new, hsa_bf16* O, int32_t* indices_out,
                                    cudaStream_t stream);

/* Number of kernels this library has launched in the calling process (all
 * devices, all streams) since it was loaded. A diagnostic counter for
 * benchmarks and tests; it is not synchronised with the GPU. */
HSA_API uint64_t hsa_kernel_launches(void);

/* Whether a bounded device-side wait has given up on the current device.
 * The tensor-core kernels (block/token scoring, attention) bound every wait
 * on an mbarrier to about two seconds of SM clock. A wait that runs out sets
 * a sticky per-device flag; the kernel then skips the work that depended on
 * the wait and runs to completion, so that launch's outputs are incomplete,
 * and while the flag stays set later waits give up early. The other entry
 * points cannot report this (they never synchronise). This call synchronises
 * the current device (cudaDeviceSynchronize), reads the flags and returns
 * HSA_ERR_TIMEOUT if one is set, else HSA_OK; HSA_ERR_CUDA on a CUDA error,
 * HSA_ERR_DEVICE on a device that is not sm_100. reset != 0 clears the flags
 * after reading them. A diagnostic for tests and benchmarks, not for the hot
 * path. */
HSA_API int hsa_device_status(int reset);

/* Test hook for the bounded-wait machinery, not for production use. The pages
 * describe no such interface. With on != 0, on the current device: every
 * bounded wait of the tensor-core kernels (block/token scoring, attention)
 * gives up after about a millisecond instead of about two seconds, and the
 * next launch of each of them loses one producer hand-off in its first CTA
 * (the scoring kernels skip producing their first tile; the attention's first
 * K-tile arrival is not made), so a consumer's wait must run out. The kernels
 * then return with incomplete outputs and hsa_device_status reports
 * HSA_ERR_TIMEOUT. Nothing faults, traps or spins without bound. With on == 0
 * the kernels behave normally again; clear the flag with
 * hsa_device_status(1) afterwards. Synchronous (cudaMemcpyToSymbol); returns
 * HSA_OK, or HSA_ERR_CUDA / HSA_ERR_DEVICE. */
HSA_API int hsa_debug_inject_lost_arrival(int on);

#ifdef __cplusplus
}
#endif
#endif /* HSA_H_ */
