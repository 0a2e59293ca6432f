// Launchers of the HISA kernels; called by the C ABI in api.cu.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "common.cuh"

namespace hsa {

// Counts kernel launches made by this library (see hsa_kernel_launches).
void count_launches(int n);

// Launches kern<<<grid, block, smem, s>>>(args...); with pdl set, as a
// programmatic dependent launch (the kernel must begin with griddep_wait()).
template <typename... KArgs, typename... Args>
inline void launch_kernel(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                          Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr;
  attr.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr.val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = &attr;
  cfg.numAttrs = pdl ? 1 : 0;
  (void)cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// 2-D row-major bf16 [rows][cols] TMA map, box {64 columns, box_rows rows},
// 128-byte swizzle. False if the driver entry point or the encoding fails.
bool make_tmap_2d(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint32_t box_rows);
int num_sms();

void launch_block_sums(const void* k_idx, int64_t Lk, int B, int d_idx, float* ksum,
                       cudaStream_t s);
void launch_select_blocks(RowMap rm, int64_t rows, const void* q_idx, const float* ksum,
                          int64_t ksum_seq_stride, int B, int m, int d_idx, int32_t* blocks,
                          int64_t max_cand, cudaStream_t s);
// max_cand: the most candidates any row can have (its keys are staged in shared memory)
void launch_select_tokens(RowMap rm, int64_t rows, const void* q_idx, const void* k_idx,
                          const int32_t* blocks, int B, int m, int k, int d_idx, int32_t* indices,
                          int64_t max_cand, cudaStream_t s);
// Tensor-core sparse attention (d = 64 or 128, any H: one launch per group of
// up to 64 heads); returns false if a launch attribute could not be set.
bool tc_attn_supported(int H, int d, int64_t Lq, int64_t Lk);
bool launch_sparse_attn_tc(int64_t Lq, const void* Q, const void* K, const void* V, const int32_t* idx,
                           int64_t Lk, int k, int H, int d, float scale, void* O, cudaStream_t s);
void launch_ksum_split(const float* ksum, int64_t n, void* split, cudaStream_t s);
bool launch_block_score_gemm(const void* q_idx, const void* bsplit, int64_t Lq, int64_t Lk, int B, int m,
                             int d_idx, int64_t nbc, uint32_t* out, int64_t ld, cudaStream_t s);
bool launch_token_score_gemm(const void* q_idx, const void* k_idx, int64_t Lq, int64_t Lk, int B, int m,
                             int d_idx, const int4* tiles, const int* ntiles, const uint32_t* pairs,
                             int64_t max_tiles, uint32_t* out, cudaStream_t s);
void launch_topm_from_keys(RowMap rm, int64_t rows, const uint32_t* bkeys, int64_t ld, int B, int m,
                           int64_t max_cand, int32_t* blocks, cudaStream_t s, bool pdl = false);
void launch_pair_lists(RowMap rm, int64_t rows, const int32_t* blocks, int B, int m, int k, int nbins,
                       int* cnt, int* off, int* cursor, int4* tiles, int* ntiles, uint32_t* pairs,
                       cudaStream_t s);
void launch_topk_from_keys(RowMap rm, int64_t rows, const int32_t* blocks, const uint32_t* tkeys, int B,
                           int m, int k, int32_t* indices, cudaStream_t s, bool pdl = false);
// (also appends each sequence's new token: k_idx/K/V rows and a completed block's sum)
void launch_decode_block_scores(int batch, int64_t capacity, const int32_t* ctx, int B, int m, int d_idx,
                                const void* q_new, const float* ksum_cache, uint32_t* bkeys, int64_t ld,
                                int d, void* k_idx_cache, void* K_cache, void* V_cache, float* ksum_w,
                                const void* k_idx_new, const void* K_new, const void* V_new, cudaStream_t s);
void launch_decode_token_scores(int batch, int64_t capacity, const int32_t* ctx, int B, int m, int d_idx,
                                const int32_t* blocks, const void* q_new, const void* k_idx_cache,
                                uint32_t* tkeys, cudaStream_t s);
// (also advances ctx: every sequence that took the step grows by one token)
void launch_decode_combine(int batch, int64_t capacity, int32_t* ctx, int H, int d, int parts,
                           const float* Opart, const float* mpart, const float* lpart, void* O, cudaStream_t s);
bool launch_sparse_attn_tc_split(int batch, const void* Q, const void* Kc, const void* Vc, const int32_t* idx,
                                 int64_t capacity, int k, int H, int d, float scale, int parts, float* Opart,
                                 float* mpart, float* lpart, cudaStream_t s, bool pdl = false);

// Sticky per-device flags set by a bounded wait that gave up (1), read on the
// host with a synchronous copy and optionally cleared; -1 on a CUDA error.
int attn_wait_flag(bool reset);
// Test hook of the tensor-core kernels on the current device: short bounded
// waits and one lost producer arrival in the next launch of CTA 0.
bool attn_set_inject(bool on);
bool score_set_inject(bool on);
int score_wait_flag(bool reset);

}  // namespace hsa
