// Oracle for hierarchical indexed sparse attention (HISA) -- TEST INFRASTRUCTURE.
//
// A plain, slow, obviously correct CPU restatement of what the GPU path
// computes. Only the test suite, the smoke check and the benchmark's CPU
// baseline may load it; the product library never does, and this file shares
// no code, header or table with the CUDA sources.
//
// Source of the method: the page "HISA: Hierarchical Indexed Sparse Attention"
// (discuz.ruhao.net thread 187), sections 第一步 (block-level coarse filter),
// 第二步 (token-level selection inside the kept blocks), the note that the
// first and last blocks are always kept, the complexity paragraph
// O(L^2/B + L*m*B), and the "drop-in replacement" paragraph (same output
// format as the original indexer, attention downstream unchanged, short
// inputs degenerate to the original method). The softmax form
// softmax(Q K^T / sqrt(d)) V over the selected keys is the one printed in the
// HiLS page's pseudocode (Step 4).
//
// Readings of points the pages leave open:
//   * scoring rule of the indexer: a plain dot product q_idx . k_idx (one
//     indexer head, no weights, no activation);
//   * block representative: the fp32 sum of the block's key rows;
//   * the m kept blocks include the two forced ones: block 0 and the query's
//     own block floor(t/B); the other m-2 are the best-scoring complete
//     blocks among 1 .. floor(t/B)-1;
//   * causal keys are j <= t (the query's own position included);
//   * ties (blocks and tokens) go to the lowest index;
//   * the k kept indices are written in ascending order, padded with -1;
//   * indexer scores are fp32 (the decision precision the GPU uses); the
//     attention is evaluated in fp64.
//
// Parity status: block sums, block selection and token selection are pinned
// by hand-worked examples, brute-force subset enumeration and the flat-top-k
// invariant; attention by closed forms and a dense textbook softmax
// reference (see tests/test_oracle.py).

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <thread>
#include <vector>

namespace {

float bf16_to_float(uint16_t bits) {
  uint32_t u = static_cast<uint32_t>(bits) << 16;
  float f;
  std::memcpy(&f, &u, sizeof f);
  return f;
}

// Run body(r) for r in [0, n) on `threads` workers (dynamic row handout).
template <class F>
void parallel_rows(int64_t n, int threads, F body) {
  if (threads <= 1 || n <= 1) {
    for (int64_t r = 0; r < n; ++r) body(r);
    return;
  }
  std::atomic<int64_t> next{0};
  std::vector<std::thread> pool;
  for (int w = 0; w < threads; ++w)
    pool.emplace_back([&] {
      for (int64_t r; (r = next.fetch_add(1)) < n;) body(r);
    });
  for (auto& th : pool) th.join();
}

// Row i of the query set has absolute position t = Lk - Lq + i.
int64_t row_of(const int64_t* rows, int64_t r) { return rows ? rows[r] : r; }

// fp32 dot product of a bf16 query row and a bf16 key row, in index order.
float dot_bf16_f32(const uint16_t* a, const uint16_t* b, int n) {
  float s = 0.0f;
  for (int c = 0; c < n; ++c) s += bf16_to_float(a[c]) * bf16_to_float(b[c]);
  return s;
}

}  // namespace

extern "C" {

// Step 1 of 第一步: representative of every complete block, ksum[b][c] =
// sum over the B rows j = b*B .. b*B+B-1 of k_idx[j][c], accumulated in fp32
// in row order. Only the floor(Lk/B) complete blocks are produced (a partial
// block is only ever the query's own block, which is kept without scoring).
int oracle_block_sums(const uint16_t* k_idx, int64_t Lk, int d_idx, int B, float* ksum) {
  if (!k_idx || !ksum || B <= 0 || d_idx <= 0 || Lk < 0) return 1;
  const int64_t nbc = Lk / B;
  for (int64_t b = 0; b < nbc; ++b)
    for (int c = 0; c < d_idx; ++c) {
      float s = 0.0f;
      for (int64_t j = b * B; j < (b + 1) * B; ++j) s += bf16_to_float(k_idx[j * d_idx + c]);
      ksum[b * d_idx + c] = s;
    }
  return 0;
}

// 第一步 block-level selection for the query rows listed in `rows` (nrows of
// them; rows == NULL means all Lq rows). Output blocks[r][0..m-1]: the kept
// block ids in ascending order, -1 padded when fewer than m exist.
//   nb = floor(t/B) + 1 causal blocks.
//   nb <= m : every causal block is kept (the short-input degeneration).
//   nb  > m : block 0 and block nb-1 (the query's own) are forced; of blocks
//             1 .. nb-2 the m-2 with the largest score q . ksum[b] are kept,
//             ordered by (score descending, block ascending).
int oracle_select_blocks(const uint16_t* q_idx, const float* ksum, int64_t Lq, int64_t Lk,
                         int d_idx, int B, int m, const int64_t* rows, int64_t nrows,
                         int32_t* blocks, int threads) {
  if (!q_idx || !ksum || !blocks || B <= 0 || m < 2 || Lq > Lk) return 1;
  parallel_rows(nrows, threads, [&](int64_t r) {
    const int64_t i = row_of(rows, r);
    const int64_t t = Lk - Lq + i;
    const int64_t nb = t / B + 1;
    int32_t* out = blocks + r * m;
    for (int s = 0; s < m; ++s) out[s] = -1;
    if (nb <= m) {
      for (int64_t b = 0; b < nb; ++b) out[b] = static_cast<int32_t>(b);
      return;
    }
    const uint16_t* q = q_idx + i * d_idx;
    std::vector<std::pair<float, int64_t>> cand;
    for (int64_t b = 1; b <= nb - 2; ++b) {
      float s = 0.0f;
      for (int c = 0; c < d_idx; ++c) s += bf16_to_float(q[c]) * ksum[b * d_idx + c];
      cand.push_back({s, b});
    }
    std::sort(cand.begin(), cand.end(), [](const auto& x, const auto& y) {
      if (x.first != y.first) return x.first > y.first;
      return x.second < y.second;
    });
    std::vector<int64_t> kept = {0, nb - 1};
    for (int s = 0; s < m - 2; ++s) kept.push_back(cand[s].second);
    std::sort(kept.begin(), kept.end());
    for (int s = 0; s < m; ++s) out[s] = static_cast<int32_t>(kept[s]);
  });
  return 0;
}

// 第二步 token-level selection. Candidates are the tokens j <= t of the kept
// blocks (blocks[r], as written by oracle_select_blocks for the same rows).
// If there are at most k candidates all are kept (the degeneration to the
// original method); otherwise the k with the largest fp32 score
// q_idx[t] . k_idx[j] are kept, ordered by (score descending, j ascending).
// Output indices[r][0..k-1] in ascending order, -1 padded.
int oracle_select_tokens(const uint16_t* q_idx, const uint16_t* k_idx, const int32_t* blocks,
                         int64_t Lq, int64_t Lk, int d_idx, int B, int m, int k,
                         const int64_t* rows, int64_t nrows, int32_t* indices, int threads) {
  if (!q_idx || !k_idx || !blocks || !indices || B <= 0 || m < 1 || k < 1 || Lq > Lk) return 1;
  parallel_rows(nrows, threads, [&](int64_t r) {
    const int64_t i = row_of(rows, r);
    const int64_t t = Lk - Lq + i;
    const uint16_t* q = q_idx + i * d_idx;
    std::vector<int64_t> cand;
    for (int s = 0; s < m; ++s) {
      const int64_t b = blocks[r * m + s];
      if (b < 0) continue;
      for (int64_t j = b * B; j < (b + 1) * B && j <= t; ++j) cand.push_back(j);
    }
    std::vector<int64_t> kept;
    if (static_cast<int64_t>(cand.size()) <= k) {
      kept = cand;
    } else {
      std::vector<std::pair<float, int64_t>> sc;
      for (int64_t j : cand) sc.push_back({dot_bf16_f32(q, k_idx + j * d_idx, d_idx), j});
      std::sort(sc.begin(), sc.end(), [](const auto& x, const auto& y) {
        if (x.first != y.first) return x.first > y.first;
        return x.second < y.second;
      });
      for (int s = 0; s < k; ++s) kept.push_back(sc[s].second);
    }
    std::sort(kept.begin(), kept.end());
    int32_t* out = indices + r * k;
    for (int s = 0; s < k; ++s)
      out[s] = s < static_cast<int>(kept.size()) ? static_cast<int32_t>(kept[s]) : -1;
  });
  return 0;
}

// Both stages for the listed rows: block sums, block selection, token
// selection. blocks_out (nrows x m) may be NULL.
int oracle_index(const uint16_t* q_idx, const uint16_t* k_idx, int64_t Lq, int64_t Lk, int d_idx,
                 int B, int m, int k, const int64_t* rows, int64_t nrows, int32_t* indices,
                 int32_t* blocks_out, int threads) {
  if (!q_idx || !k_idx || !indices || B <= 0 || d_idx <= 0) return 1;
  std::vector<float> ksum(static_cast<size_t>(Lk / B) * d_idx + 1);
  if (oracle_block_sums(k_idx, Lk, d_idx, B, ksum.data())) return 1;
  std::vector<int32_t> blocks(static_cast<size_t>(nrows) * m + 1);
  if (oracle_select_blocks(q_idx, ksum.data(), Lq, Lk, d_idx, B, m, rows, nrows, blocks.data(),
                           threads))
    return 1;
  if (blocks_out) std::memcpy(blocks_out, blocks.data(), sizeof(int32_t) * nrows * m);
  return oracle_select_tokens(q_idx, k_idx, blocks.data(), Lq, Lk, d_idx, B, m, k, rows, nrows,
                              indices, threads);
}

// Exact softmax attention over the selected keys, shared by all H heads
// (multi-query attention: one K/V head). For query row i and head h:
//   x_j = scale * sum_c Q[i][h][c] * K[j][c]     for j in indices[r] (j >= 0)
//   O[r][h][:] = sum_j exp(x_j - max x) V[j][:] / sum_j exp(x_j - max x)
// evaluated in fp64. A row with no valid index yields zeros.
int oracle_sparse_attn(const uint16_t* Q, const uint16_t* K, const uint16_t* V,
                       const int32_t* indices, int64_t Lq, int64_t Lk, int H, int d, int k,
                       double scale, const int64_t* rows, int64_t nrows, double* O, int threads) {
  if (!Q || !K || !V || !indices || !O || H <= 0 || d <= 0 || k < 1) return 1;
  parallel_rows(nrows, threads, [&](int64_t r) {
    const int64_t i = row_of(rows, r);
    const int32_t* idx = indices + r * k;
    std::vector<int64_t> S;
    for (int s = 0; s < k; ++s)
      if (idx[s] >= 0 && idx[s] < Lk) S.push_back(idx[s]);
    std::vector<double> x(S.size());
    for (int h = 0; h < H; ++h) {
      const uint16_t* q = Q + (i * H + h) * static_cast<int64_t>(d);
      double* o = O + (r * H + h) * static_cast<int64_t>(d);
      for (int c = 0; c < d; ++c) o[c] = 0.0;
      if (S.empty()) continue;
      double mx = -INFINITY;
      for (size_t a = 0; a < S.size(); ++a) {
        double s = 0.0;
        for (int c = 0; c < d; ++c)
          s += static_cast<double>(bf16_to_float(q[c])) * bf16_to_float(K[S[a] * d + c]);
        x[a] = s * scale;
        mx = std::max(mx, x[a]);
      }
      double l = 0.0;
      for (size_t a = 0; a < S.size(); ++a) {
        const double p = std::exp(x[a] - mx);
        l += p;
        for (int c = 0; c < d; ++c) o[c] += p * bf16_to_float(V[S[a] * d + c]);
      }
      for (int c = 0; c < d; ++c) o[c] /= l;
    }
  });
  return 0;
}

}  // extern "C"
