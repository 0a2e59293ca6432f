// hsa_prefill_host: the whole path (index, then sparse attention) for queries
// whose inputs and outputs live in host memory, with the host<->device copies
// overlapped with the kernels. The indices go out as soon as the indexer is
// done; the query rows are cut into chunks, and while the attention of chunk
// c runs, chunk c+1's Q rows come in and chunk c-1's O rows go out, on two
// copy streams of the library's own that fork from the caller's stream and
// join back into it. (The device-to-host direction, O and the indices, is the
// larger: starting it with the indices keeps it busy from the indexer on.)
#include <algorithm>
#include <mutex>

#include "hsa.h"
#include "kernels.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxChunks = 16;
constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// A device's copy streams and the events that order them, created on the
// device's first call and kept until the process exits.
struct CopyStreams {
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaEvent_t start = nullptr, joined = nullptr, idx_ready = nullptr;
  cudaEvent_t q_ready[kMaxChunks] = {}, o_ready[kMaxChunks] = {};
  std::mutex mu;  // one call at a time enqueues on them
  bool ok = false;
};
CopyStreams g_copy[kMaxDevices];
std::mutex g_copy_init;

CopyStreams* copy_streams() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(g_copy_init);
  CopyStreams& c = g_copy[dev];
  if (!c.ok) {
    const unsigned f = cudaEventDisableTiming;
    bool good = cudaStreamCreateWithFlags(&c.h2d, cudaStreamNonBlocking) == cudaSuccess &&
                cudaStreamCreateWithFlags(&c.d2h, cudaStreamNonBlocking) == cudaSuccess &&
                cudaEventCreateWithFlags(&c.start, f) == cudaSuccess &&
                cudaEventCreateWithFlags(&c.joined, f) == cudaSuccess &&
                cudaEventCreateWithFlags(&c.idx_ready, f) == cudaSuccess;
    for (int i = 0; good && i < kMaxChunks; ++i)
      good = cudaEventCreateWithFlags(&c.q_ready[i], f) == cudaSuccess &&
             cudaEventCreateWithFlags(&c.o_ready[i], f) == cudaSuccess;
    if (!good) return nullptr;
    c.ok = true;
  }
  return &c;
}

// Device workspace (256-byte aligned regions): the device copies of the
// inputs and outputs, then the indexer's own workspace.
struct HostWs {
  size_t q_idx, k_idx, Q, K, V, O, idx, index_ws, index_ws_bytes, total;
};
int host_ws(const hsa_params* p, int64_t Lq, int64_t Lk, HostWs* w) {
  size_t iw = 0;
  if (int e = hsa_index_workspace_size(p, Lq, Lk, &iw)) return e;
  // the attention's own checks (H, d, k, scale, Lk); with no query nothing runs
  if (int e = hsa_sparse_attn(p, 0, Lk, nullptr, nullptr, nullptr, nullptr, nullptr, nullptr)) return e;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o += align_up(bytes > 0 ? bytes : 1); return at; };
  w->q_idx = take(size_t(Lq) * p->d_idx * 2);
  w->k_idx = take(size_t(Lk) * p->d_idx * 2);
  w->Q = take(size_t(Lq) * p->H * p->d * 2);
  w->K = take(size_t(Lk) * p->d * 2);
  w->V = take(size_t(Lk) * p->d * 2);
  w->O = take(size_t(Lq) * p->H * p->d * 2);
  w->idx = take(size_t(Lq) * p->k * 4);
  w->index_ws_bytes = iw;
  w->index_ws = take(iw);
  w->total = o;
  return HSA_OK;
}

// Rows [r0, r0 + rows) of chunk c when Lq query rows are cut into n chunks
// of whole 128-row tiles (the last chunk takes the ragged tail).
void chunk_rows(int64_t Lq, int n, int c, int64_t* r0, int64_t* rows) {
  const int64_t tiles = (Lq + 127) / 128;
  const int64_t per = (tiles + n - 1) / n * 128;
  *r0 = std::min<int64_t>(Lq, int64_t(c) * per);
  *rows = std::min<int64_t>(Lq, *r0 + per) - *r0;
}

}  // namespace

extern "C" {

int hsa_prefill_host_workspace_size(const hsa_params* p, int64_t Lq, int64_t Lk, size_t* bytes) {
  if (!bytes) return HSA_ERR_ARG;
  HostWs w{};
  if (int e = host_ws(p, Lq, Lk, &w)) return e;
  *bytes = w.total;
  return HSA_OK;
}

int hsa_prefill_host(const hsa_params* p, int64_t Lq, int64_t Lk, const hsa_bf16* q_idx_h,
                     const hsa_bf16* k_idx_h, const hsa_bf16* Q_h, const hsa_bf16* K_h,
                     const hsa_bf16* V_h, hsa_bf16* O_h, int32_t* indices_h, void* workspace,
                     size_t workspace_bytes, cudaStream_t stream) {
  HostWs w{};
  if (int e = host_ws(p, Lq, Lk, &w)) return e;
  if (Lq == 0) return HSA_OK;
  if (!q_idx_h || !k_idx_h || !Q_h || !K_h || !V_h || !O_h) return HSA_ERR_ARG;
  if (!workspace || (reinterpret_cast<uintptr_t>(workspace) & (kAlign - 1)) || workspace_bytes < w.total)
    return HSA_ERR_WORKSPACE;
  CopyStreams* cs = copy_streams();
  if (!cs) return HSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(cs->mu);
  char* ws = static_cast<char*>(workspace);
  hsa_bf16* q_idx = reinterpret_cast<hsa_bf16*>(ws + w.q_idx);
  hsa_bf16* k_idx = reinterpret_cast<hsa_bf16*>(ws + w.k_idx);
  hsa_bf16* Q = reinterpret_cast<hsa_bf16*>(ws + w.Q);
  hsa_bf16* K = reinterpret_cast<hsa_bf16*>(ws + w.K);
  hsa_bf16* V = reinterpret_cast<hsa_bf16*>(ws + w.V);
  hsa_bf16* O = reinterpret_cast<hsa_bf16*>(ws + w.O);
  int32_t* idx = reinterpret_cast<int32_t*>(ws + w.idx);
  const size_t qrow = size_t(p->H) * p->d;  // elements of one query's Q or O row
  const int n = int(std::min<int64_t>(kMaxChunks, (Lq + 127) / 128));
  bool ok = true;
  int status = HSA_OK;
  auto cu = [&](cudaError_t e) { ok = ok && e == cudaSuccess; };
  // fork: both copy streams start after the caller's earlier work
  cu(cudaEventRecord(cs->start, stream));
  cu(cudaStreamWaitEvent(cs->h2d, cs->start, 0));
  cu(cudaStreamWaitEvent(cs->d2h, cs->start, 0));
  if (ok) {
    // the indexer's inputs on the caller's stream, then the indexer
    cu(cudaMemcpyAsync(k_idx, k_idx_h, size_t(Lk) * p->d_idx * 2, cudaMemcpyHostToDevice, stream));
    cu(cudaMemcpyAsync(q_idx, q_idx_h, size_t(Lq) * p->d_idx * 2, cudaMemcpyHostToDevice, stream));
    if (ok) status = hsa_index(p, Lq, Lk, q_idx, k_idx, idx, ws + w.index_ws, w.index_ws_bytes, stream);
    // the indices out on the D2H stream, while the attention runs
    if (ok && status == HSA_OK && indices_h) {
      cu(cudaEventRecord(cs->idx_ready, stream));
      cu(cudaStreamWaitEvent(cs->d2h, cs->idx_ready, 0));
      cu(cudaMemcpyAsync(indices_h, idx, size_t(Lq) * p->k * 4, cudaMemcpyDeviceToHost, cs->d2h));
    }
  }
  if (ok && status == HSA_OK) {
    // the attention's inputs on the H2D stream: K and V, then Q chunk by chunk
    cu(cudaMemcpyAsync(K, K_h, size_t(Lk) * p->d * 2, cudaMemcpyHostToDevice, cs->h2d));
    cu(cudaMemcpyAsync(V, V_h, size_t(Lk) * p->d * 2, cudaMemcpyHostToDevice, cs->h2d));
    for (int c = 0; c < n; ++c) {
      int64_t r0, rows;
      chunk_rows(Lq, n, c, &r0, &rows);
      cu(cudaMemcpyAsync(Q + r0 * qrow, Q_h + r0 * qrow, size_t(rows) * qrow * 2, cudaMemcpyHostToDevice,
                         cs->h2d));
      cu(cudaEventRecord(cs->q_ready[c], cs->h2d));
    }
    // the attention of each chunk on the caller's stream, after its Q rows
    for (int c = 0; c < n && ok && status == HSA_OK; ++c) {
      int64_t r0, rows;
      chunk_rows(Lq, n, c, &r0, &rows);
      cu(cudaStreamWaitEvent(stream, cs->q_ready[c], 0));
      if (ok && rows > 0)
        status = hsa_sparse_attn(p, rows, Lk, Q + r0 * qrow, K, V, idx + r0 * p->k, O + r0 * qrow, stream);
      cu(cudaEventRecord(cs->o_ready[c], stream));
    }
  }
  if (ok && status == HSA_OK) {
    // each chunk's O rows out on the D2H stream as soon as its attention is done
    for (int c = 0; c < n; ++c) {
      int64_t r0, rows;
      chunk_rows(Lq, n, c, &r0, &rows);
      cu(cudaStreamWaitEvent(cs->d2h, cs->o_ready[c], 0));
      cu(cudaMemcpyAsync(O_h + r0 * qrow, O + r0 * qrow, size_t(rows) * qrow * 2, cudaMemcpyDeviceToHost,
                         cs->d2h));
    }
  }
  // join, after a failure too: the caller's stream goes on only once every
  // copy enqueued above has finished
  bool joined = cudaEventRecord(cs->joined, cs->d2h) == cudaSuccess &&
                cudaStreamWaitEvent(stream, cs->joined, 0) == cudaSuccess;
  joined = joined && cudaEventRecord(cs->joined, cs->h2d) == cudaSuccess &&
           cudaStreamWaitEvent(stream, cs->joined, 0) == cudaSuccess;
  if (status != HSA_OK) return status;
  return ok && joined ? HSA_OK : HSA_ERR_CUDA;
}

}  // extern "C"
