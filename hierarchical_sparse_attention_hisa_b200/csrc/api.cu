// C ABI of libhsa.so (declared in include/hsa.h): host-side argument checks,
// workspace layout and kernel launches. No allocation, no synchronisation.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "hsa.h"
#include "kernels.cuh"

namespace hsa {
static std::atomic<uint64_t> g_launches{0};
void count_launches(int n) { g_launches.fetch_add(uint64_t(n), std::memory_order_relaxed); }
}  // namespace hsa

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Blocks of a sequence the block stage scores per query.
constexpr int64_t kMaxBlocks = 16384;
// Token candidates per query (kept blocks x B): the tensor-core token scoring
// with its key-stream top-k takes up to kMaxCandidates, the CUDA-core token
// scoring (block sizes the MMA cannot take) stages them in shared memory and
// takes up to kMaxCandidatesSmem.
constexpr int64_t kMaxCandidates = 65536;
constexpr int64_t kMaxCandidatesSmem = 16384;
constexpr int kMaxM = 512;  // kept blocks per query

int check_device() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return HSA_ERR_CUDA;
  thread_local int cached_dev = -1, cached_ok = 0;  // per host thread: no shared mutable state
  if (dev != cached_dev) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
      return HSA_ERR_CUDA;
    cached_ok = major == 10;
    cached_dev = dev;
  }
  return cached_ok ? HSA_OK : HSA_ERR_DEVICE;
}

int check_index_params(const hsa_params* p) {
  if (!p) return HSA_ERR_ARG;
  if (p->B < 1 || p->B > 1024) return HSA_ERR_ARG;
  if (p->m < 2 || p->m > kMaxM) return HSA_ERR_ARG;
  if (p->k < 1 || p->k > 8192) return HSA_ERR_ARG;
  if (p->d_idx != 64 && p->d_idx != 128) return HSA_ERR_ARG;
  const bool mma_tokens = p->B == 64 || p->B == 128 || p->B == 256;
  if (int64_t(p->m) * p->B > (mma_tokens ? kMaxCandidates : kMaxCandidatesSmem)) return HSA_ERR_ARG;
  return HSA_OK;
}

int check_attn_params(const hsa_params* p) {
  if (!p) return HSA_ERR_ARG;
  if (p->k < 1 || p->k > 8192) return HSA_ERR_ARG;
  if (p->H < 1 || p->H > 128) return HSA_ERR_ARG;
  if (p->d != 64 && p->d != 128) return HSA_ERR_ARG;
  if (!(p->scale >= 0.f) || std::isinf(p->scale)) return HSA_ERR_ARG;
  return HSA_OK;
}

float softmax_scale(const hsa_params* p) {
  return p->scale > 0.f ? p->scale : 1.0f / std::sqrt(float(p->d));
}

int check_lengths(const hsa_params* p, int64_t Lq, int64_t Lk) {
  if (Lq < 0 || Lk < 1 || Lq > Lk || Lq > (int64_t(1) << 31) - 1) return HSA_ERR_ARG;
  if (Lk > (int64_t(1) << 31) - 1) return HSA_ERR_ARG;
  if (Lk / p->B > kMaxBlocks) return HSA_ERR_ARG;
  return HSA_OK;
}

int launch_status() {
  return cudaGetLastError() == cudaSuccess ? HSA_OK : HSA_ERR_CUDA;
}

// Largest number of block candidates any query of [Lk-Lq, Lk) scores.
int64_t max_block_candidates(const hsa_params* p, int64_t Lk) {
  const int64_t nb = (Lk - 1) / p->B + 1;
  return nb > 2 ? nb - 2 : 1;
}

// Workspace of the indexer (all offsets 256-byte aligned):
//   ksum   [nbc][d_idx] fp32          block sums
//   bsplit [3][nbc][d_idx] bf16       hi/mid/lo planes of ksum
//   bkeys  [Lq][ldb] u32              block-score keys (ldb = nbc rounded to 64)
//   blocks [Lq][m] i32                kept blocks
//   cnt/cursor [nbins] i32            pairs per key block (nbins = ceil(Lk/B))
//   off [2][nbins] i32                first pair and first tile of each key block
//   ntiles i32, tiles [max_tiles] int4, pairs [Lq*m] u32
//   tkeys  [Lq][m][B] u32             token-score keys
struct IndexWs {
  size_t ksum, bsplit, bkeys, blocks, cnt, off, cursor, ntiles, tiles, pairs, tkeys, total;
  int64_t nbc, ldb, nbins, max_tiles;
};
IndexWs index_ws(const hsa_params* p, int64_t Lq, int64_t Lk) {
  IndexWs w{};
  w.nbc = Lk / p->B;
  w.ldb = (w.nbc + 63) / 64 * 64;
  w.nbins = (Lk + p->B - 1) / p->B;
  w.max_tiles = (Lq * p->m + 127) / 128 + w.nbins;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o += align_up(bytes > 0 ? bytes : 1); return at; };
  w.ksum = take(size_t(w.nbc) * p->d_idx * 4);
  w.bsplit = take(size_t(3) * w.nbc * p->d_idx * 2);
  w.bkeys = take(size_t(Lq) * w.ldb * 4);
  w.blocks = take(size_t(Lq) * p->m * 4);
  w.cnt = take(size_t(w.nbins) * 4);
  w.off = take(size_t(w.nbins) * 8);
  w.cursor = take(size_t(w.nbins) * 4);
  w.ntiles = take(16);
  w.tiles = take(size_t(w.max_tiles) * 16);
  w.pairs = take(size_t(Lq) * p->m * 4);
  w.tkeys = take(size_t(Lq) * p->m * p->B * 4);
  w.total = o;
  return w;
}

// Tensor-core scoring covers d_idx in {64, 128}; block scoring needs a full
// 128-query tile and at least 64 rows of split block sums, token scoring a
// block size the MMA N dimension can take and one full key block.
bool block_gemm_ok(const hsa_params* p, int64_t Lq, int64_t Lk) {
  return Lq >= 128 && 3 * (Lk / p->B) >= 64;
}
bool token_gemm_ok(const hsa_params* p, int64_t Lq, int64_t Lk) {
  return (p->B == 64 || p->B == 128 || p->B == 256) && Lk >= p->B && Lq * int64_t(p->m) < (int64_t(1) << 32);
}

// Kept blocks for rows [0, Lq) from fp32 block sums.
void run_select_blocks(const hsa_params* p, int64_t Lq, int64_t Lk, const void* q_idx, const float* ksum,
                       int32_t* blocks, char* ws, const IndexWs& w, cudaStream_t s, bool* ok) {
  hsa::RowMap rm{Lq, Lk, nullptr, 0};
  const int64_t nb_last = (Lk - 1) / p->B + 1;
  if (nb_last > p->m && p->m > 2 && block_gemm_ok(p, Lq, Lk)) {
    void* bsplit = ws + w.bsplit;
    uint32_t* bkeys = reinterpret_cast<uint32_t*>(ws + w.bkeys);
    hsa::launch_ksum_split(ksum, w.nbc * p->d_idx, bsplit, s);
    if (!hsa::launch_block_score_gemm(q_idx, bsplit, Lq, Lk, p->B, p->m, p->d_idx, w.nbc, bkeys, w.ldb, s)) {
      *ok = false;
      return;
    }
    hsa::launch_topm_from_keys(rm, Lq, bkeys, w.ldb, p->B, p->m, max_block_candidates(p, Lk), blocks, s, true);
  } else {
    hsa::launch_select_blocks(rm, Lq, q_idx, ksum, 0, p->B, p->m, p->d_idx, blocks,
                              max_block_candidates(p, Lk), s);
  }
}

// Kept tokens for rows [0, Lq) from their kept blocks.
void run_select_tokens(const hsa_params* p, int64_t Lq, int64_t Lk, const void* q_idx, const void* k_idx,
                       const int32_t* blocks, int32_t* indices, char* ws, const IndexWs& w, cudaStream_t s,
                       bool* ok) {
  hsa::RowMap rm{Lq, Lk, nullptr, 0};
  if (token_gemm_ok(p, Lq, Lk)) {
    int* cnt = reinterpret_cast<int*>(ws + w.cnt);
    int* off = reinterpret_cast<int*>(ws + w.off);
    int* cursor = reinterpret_cast<int*>(ws + w.cursor);
    int* ntiles = reinterpret_cast<int*>(ws + w.ntiles);
    int4* tiles = reinterpret_cast<int4*>(ws + w.tiles);
    uint32_t* pairs = reinterpret_cast<uint32_t*>(ws + w.pairs);
    uint32_t* tkeys = reinterpret_cast<uint32_t*>(ws + w.tkeys);
    hsa::launch_pair_lists(rm, Lq, blocks, p->B, p->m, p->k, int(w.nbins), cnt, off, cursor, tiles, ntiles,
                           pairs, s);
    if (!hsa::launch_token_score_gemm(q_idx, k_idx, Lq, Lk, p->B, p->m, p->d_idx, tiles, ntiles, pairs,
                                      w.max_tiles, tkeys, s)) {
      *ok = false;
      return;
    }
    hsa::launch_topk_from_keys(rm, Lq, blocks, tkeys, p->B, p->m, p->k, indices, s, true);
  } else {
    // CUDA-core scoring: the row's candidates (at most m*B, at most Lk) in shared memory
    if (std::min<int64_t>(int64_t(p->m) * p->B, Lk) > kMaxCandidatesSmem) {
      *ok = false;
      return;
    }
    hsa::launch_select_tokens(rm, Lq, q_idx, k_idx, blocks, p->B, p->m, p->k, p->d_idx, indices,
                              std::min<int64_t>(int64_t(p->m) * p->B, Lk), s);
  }
}


}  // namespace

extern "C" {

uint64_t hsa_kernel_launches(void) { return hsa::g_launches.load(std::memory_order_relaxed); }

int hsa_device_status(int reset) {
  if (int e = check_device()) return e;
  if (cudaDeviceSynchronize() != cudaSuccess) return HSA_ERR_CUDA;
  const int a = hsa::attn_wait_flag(reset != 0);
  const int b = hsa::score_wait_flag(reset != 0);
  if (a < 0 || b < 0) return HSA_ERR_CUDA;
  return a || b ? HSA_ERR_TIMEOUT : HSA_OK;
}

int hsa_debug_inject_lost_arrival(int on) {
  if (int e = check_device()) return e;
  if (!hsa::attn_set_inject(on != 0) || !hsa::score_set_inject(on != 0)) return HSA_ERR_CUDA;
  return HSA_OK;
}

const char* hsa_status_string(int status) {
  switch (status) {
    case HSA_OK: return "ok";
    case HSA_ERR_ARG: return "invalid argument (null/misaligned pointer or unsupported size)";
    case HSA_ERR_WORKSPACE: return "workspace missing or too small";
    case HSA_ERR_CUDA: return "CUDA launch or runtime error";
    case HSA_ERR_TIMEOUT: return "bounded device wait gave up";
    case HSA_ERR_DEVICE: return "current device is not an sm_100 (B200-class) GPU";
    default: return "unknown status";
  }
}

int hsa_index_workspace_size(const hsa_params* p, int64_t Lq, int64_t Lk, size_t* bytes) {
  if (!bytes) return HSA_ERR_ARG;
  if (int e = check_index_params(p)) return e;
  if (int e = check_lengths(p, Lq, Lk)) return e;
  *bytes = index_ws(p, Lq, Lk).total;
  return HSA_OK;
}

int hsa_block_sums(const hsa_params* p, int64_t Lk, const hsa_bf16* k_idx, float* ksum,
                   cudaStream_t stream) {
  if (int e = check_index_params(p)) return e;
  if (Lk < 0) return HSA_ERR_ARG;
  if (Lk / p->B == 0) return HSA_OK;
  if (!aligned16(k_idx) || !aligned16(ksum)) return HSA_ERR_ARG;
  if (int e = check_device()) return e;
  hsa::launch_block_sums(k_idx, Lk, p->B, p->d_idx, ksum, stream);
  return launch_status();
}

int hsa_select_blocks(const hsa_params* p, int64_t Lq, int64_t Lk, const hsa_bf16* q_idx,
                      const float* ksum, int32_t* blocks, void* workspace,
                      size_t workspace_bytes, cudaStream_t stream) {
  if (int e = check_index_params(p)) return e;
  if (int e = check_lengths(p, Lq, Lk)) return e;
  if (Lq == 0) return HSA_OK;
  if (!aligned16(q_idx) || !aligned16(blocks) || (Lk / p->B > 0 && !aligned16(ksum)))
    return HSA_ERR_ARG;
  const IndexWs w = index_ws(p, Lq, Lk);
  if (!aligned16(workspace) || workspace_bytes < w.total) return HSA_ERR_WORKSPACE;
  if (int e = check_device()) return e;
  bool ok = true;
  run_select_blocks(p, Lq, Lk, q_idx, ksum, blocks, static_cast<char*>(workspace), w, stream, &ok);
  return ok ? launch_status() : HSA_ERR_CUDA;
}

int hsa_select_tokens(const hsa_params* p, int64_t Lq, int64_t Lk, const hsa_bf16* q_idx,
                      const hsa_bf16* k_idx, const int32_t* blocks, int32_t* indices,
                      void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (int e = check_index_params(p)) return e;
  if (int e = check_lengths(p, Lq, Lk)) return e;
  if (Lq == 0) return HSA_OK;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(blocks) || !aligned16(indices))
    return HSA_ERR_ARG;
  const IndexWs w = index_ws(p, Lq, Lk);
  if (!aligned16(workspace) || workspace_bytes < w.total) return HSA_ERR_WORKSPACE;
  if (int e = check_device()) return e;
  bool ok = true;
  run_select_tokens(p, Lq, Lk, q_idx, k_idx, blocks, indices, static_cast<char*>(workspace), w, stream, &ok);
  return ok ? launch_status() : HSA_ERR_CUDA;
}

int hsa_index(const hsa_params* p, int64_t Lq, int64_t Lk, const hsa_bf16* q_idx,
              const hsa_bf16* k_idx, int32_t* indices, void* workspace, size_t workspace_bytes,
              cudaStream_t stream) {
  if (int e = check_index_params(p)) return e;
  if (int e = check_lengths(p, Lq, Lk)) return e;
  if (Lq == 0) return HSA_OK;
  if (!aligned16(q_idx) || !aligned16(k_idx) || !aligned16(indices)) return HSA_ERR_ARG;
  const IndexWs w = index_ws(p, Lq, Lk);
  if (!aligned16(workspace) || workspace_bytes < w.total) return HSA_ERR_WORKSPACE;
  if (int e = check_device()) return e;
  char* ws = static_cast<char*>(workspace);
  float* ksum = reinterpret_cast<float*>(ws + w.ksum);
  int32_t* blocks = reinterpret_cast<int32_t*>(ws + w.blocks);
  bool ok = true;
  hsa::launch_block_sums(k_idx, Lk, p->B, p->d_idx, ksum, stream);
  run_select_blocks(p, Lq, Lk, q_idx, ksum, blocks, ws, w, stream, &ok);
  if (ok) run_select_tokens(p, Lq, Lk, q_idx, k_idx, blocks, indices, ws, w, stream, &ok);
  return ok ? launch_status() : HSA_ERR_CUDA;
}

int hsa_sparse_attn(const hsa_params* p, int64_t Lq, int64_t Lk, const hsa_bf16* Q,
                    const hsa_bf16* K, const hsa_bf16* V, const int32_t* indices, hsa_bf16* O,
                    cudaStream_t stream) {
  if (int e = check_attn_params(p)) return e;
  if (Lq < 0 || Lk < 1 || Lq > (int64_t(1) << 31) - 1 || Lk > (int64_t(1) << 31) - 1)
    return HSA_ERR_ARG;
  if (Lq == 0) return HSA_OK;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(indices) || !aligned16(O))
    return HSA_ERR_ARG;
  if (int e = check_device()) return e;
  if (!hsa::tc_attn_supported(p->H, p->d, Lq, Lk)) return HSA_ERR_ARG;
  if (!hsa::launch_sparse_attn_tc(Lq, Q, K, V, indices, Lk, p->k, p->H, p->d, softmax_scale(p), O, stream))
    return HSA_ERR_CUDA;
  return launch_status();
}

}  // extern "C"

namespace {

// Workspace of a decode step (256-byte aligned regions):
//   blocks [batch][m] i32, indices [batch][k] i32 (unless the caller takes them),
//   block-score keys [batch][capacity/B] u32, token-score keys [batch][m*B] u32,
//   attention parts: O [batch*parts][H][d] f32, maxima and row sums [batch*parts][H] f32.
struct DecodeWs {
  size_t blocks, idx, bkeys, tkeys, opart, mpart, lpart, total;
  int parts;
};
DecodeWs decode_ws(const hsa_params* p, int32_t batch, int64_t capacity) {
  DecodeWs w{};
  const int tiles = (p->k + 127) / 128;
  // enough parts per query to give every SM work at small batch, at most 16
  // (the combine kernel holds every part's values in registers)
  w.parts = batch > 0 ? std::max(1, std::min(std::min(tiles, 16), 128 / std::max(1, int(batch)))) : 1;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o += align_up(bytes > 0 ? bytes : 1); return at; };
  w.blocks = take(size_t(batch) * p->m * 4);
  w.idx = take(size_t(batch) * p->k * 4);
  w.bkeys = take(size_t(batch) * (capacity / p->B) * 4);
  w.tkeys = take(size_t(batch) * p->m * p->B * 4);
  w.opart = take(size_t(batch) * w.parts * p->H * p->d * 4);
  w.mpart = take(size_t(batch) * w.parts * p->H * 4);
  w.lpart = take(size_t(batch) * w.parts * p->H * 4);
  w.total = o;
  return w;
}

}  // namespace

extern "C" {

int hsa_decode_workspace_size(const hsa_params* p, int32_t batch, int64_t capacity,
                              size_t* bytes) {
  if (!bytes) return HSA_ERR_ARG;
  if (int e = check_index_params(p)) return e;
  if (int e = check_attn_params(p)) return e;
  if (batch < 0 || capacity < p->B || capacity % p->B) return HSA_ERR_ARG;
  *bytes = decode_ws(p, batch, capacity).total;
  return HSA_OK;
}

int hsa_decode_step(const hsa_params* p, int32_t batch, int64_t capacity, int32_t* ctx_len,
                    hsa_bf16* k_idx_cache, hsa_bf16* K_cache, hsa_bf16* V_cache,
                    float* ksum_cache, const hsa_bf16* q_idx_new, const hsa_bf16* k_idx_new,
                    const hsa_bf16* Q_new, const hsa_bf16* K_new, const hsa_bf16* V_new,
                    hsa_bf16* O, int32_t* indices_out, void* workspace, size_t workspace_bytes,
                    cudaStream_t stream) {
  size_t need = 0;
  if (int e = hsa_decode_workspace_size(p, batch, capacity, &need)) return e;
  if (capacity / p->B > kMaxBlocks || capacity > (int64_t(1) << 31) - 1) return HSA_ERR_ARG;
  if (batch == 0) return HSA_OK;
  const void* ptrs[] = {k_idx_cache, K_cache, V_cache, ksum_cache, q_idx_new,
                        k_idx_new, Q_new, K_new, V_new, O};
  for (const void* q : ptrs)
    if (!aligned16(q)) return HSA_ERR_ARG;
  if (!ctx_len || (reinterpret_cast<uintptr_t>(ctx_len) & 3u)) return HSA_ERR_ARG;
  if (indices_out && !aligned16(indices_out)) return HSA_ERR_ARG;
  if (!aligned16(workspace) || workspace_bytes < need) return HSA_ERR_WORKSPACE;
  if (int e = check_device()) return e;
  const DecodeWs w = decode_ws(p, batch, capacity);
  char* ws = static_cast<char*>(workspace);
  int32_t* blocks = reinterpret_cast<int32_t*>(ws + w.blocks);
  int32_t* idx = indices_out ? indices_out : reinterpret_cast<int32_t*>(ws + w.idx);
  uint32_t* bkeys = reinterpret_cast<uint32_t*>(ws + w.bkeys);
  uint32_t* tkeys = reinterpret_cast<uint32_t*>(ws + w.tkeys);
  const int64_t nbc = capacity / p->B;
  hsa::RowMap rm{batch, capacity, ctx_len, capacity};
  // The step's kernels are programmatic dependent launches: each may begin
  // launching while its predecessor runs, and waits for it before touching
  // memory (griddepcontrol), which hides the launch gaps of a short step.
  // 1. append the new token (and the block sum of a block it completes), in
  //    the same kernel as 2. the block scores against the block-sum cache;
  //    top-m with the forced blocks
  hsa::launch_decode_block_scores(batch, capacity, ctx_len, p->B, p->m, p->d_idx, q_idx_new, ksum_cache,
                                  bkeys, nbc, p->d, k_idx_cache, K_cache, V_cache, ksum_cache, k_idx_new,
                                  K_new, V_new, stream);
  hsa::launch_topm_from_keys(rm, batch, bkeys, nbc, p->B, p->m, nbc > 2 ? nbc - 2 : 1, blocks, stream, true);
  // 3. token scores inside the kept blocks, top-k
  hsa::launch_decode_token_scores(batch, capacity, ctx_len, p->B, p->m, p->d_idx, blocks, q_idx_new,
                                  k_idx_cache, tkeys, stream);
  hsa::launch_topk_from_keys(rm, batch, blocks, tkeys, p->B, p->m, p->k, idx, stream, true);
  // 4. attention over the kept tokens: parts of each query on the tensor cores,
  //    then combined; 5. the combine also grows each sequence by one token
  if (!hsa::tc_attn_supported(p->H, p->d, batch, capacity)) return HSA_ERR_ARG;
  float* opart = reinterpret_cast<float*>(ws + w.opart);
  float* mpart = reinterpret_cast<float*>(ws + w.mpart);
  float* lpart = reinterpret_cast<float*>(ws + w.lpart);
  if (!hsa::launch_sparse_attn_tc_split(batch, Q_new, K_cache, V_cache, idx, capacity, p->k, p->H, p->d,
                                        softmax_scale(p), w.parts, opart, mpart, lpart, stream, true))
    return HSA_ERR_CUDA;
  hsa::launch_decode_combine(batch, capacity, ctx_len, p->H, p->d, w.parts, opart, mpart, lpart, O, stream);
  return launch_status();
}

}  // extern "C"
