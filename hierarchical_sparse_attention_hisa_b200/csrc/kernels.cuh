// Launchers of the HISA kernels; called by the C ABI in api.cu.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "common.cuh"

namespace hsa {

// Counts kernel launches made by this library (see hsa_kernel_launches).
void count_launches(int n);

void launch_block_sums(const void* k_idx, int64_t Lk, int B, int d_idx, float* ksum,
                       cudaStream_t s);
void launch_select_blocks(RowMap rm, int64_t rows, const void* q_idx, const float* ksum,
                          int64_t ksum_seq_stride, int B, int m, int d_idx, int32_t* blocks,
                          int64_t max_cand, cudaStream_t s);
void launch_select_tokens(RowMap rm, int64_t rows, const void* q_idx, const void* k_idx,
                          const int32_t* blocks, int B, int m, int k, int d_idx, int32_t* indices,
                          cudaStream_t s);
void launch_sparse_attn_simple(RowMap rm, int64_t rows, const void* Q, const void* K, const void* V,
                               const int32_t* idx, int k, int H, int d, float scale, void* O,
                               cudaStream_t s);
// Tensor-core sparse attention (d = 128, 1 <= H <= 64); returns false if a
// tensor map or launch attribute could not be set up.
bool tc_attn_supported(int H, int d, int64_t Lq, int64_t Lk);
bool launch_sparse_attn_tc(int64_t Lq, const void* Q, const void* K, const void* V, const int32_t* idx,
                           int64_t Lk, int k, int H, float scale, void* O, cudaStream_t s);
void launch_decode_append(int batch, int64_t capacity, const int32_t* ctx, int B, int d_idx, int d,
                          void* k_idx_cache, void* K_cache, void* V_cache, float* ksum_cache,
                          const void* k_idx_new, const void* K_new, const void* V_new,
                          cudaStream_t s);
void launch_decode_advance(int batch, int64_t capacity, int32_t* ctx, cudaStream_t s);

}  // namespace hsa
