// Indexer scoring on tcgen05 tensor cores: the two dense contractions of the
// HISA indexer (page "HISA: Hierarchical Indexed Sparse Attention",
// sections 第一步 and 第二步), written out as order-preserving uint32 keys
// for the radix selections that follow.
//
//   block scores   S[i][b] = q_idx[i] . ksum[b]     A = 128 query rows (tiled),
//                  ksum split into three bf16 planes hi + mid + lo (exact for
//                  |ksum| < 2^24 with at most 24 significant bits), so three
//                  bf16 MMAs accumulate the fp32 result;
//   token scores   S[i][s][c] = q_idx[i] . k_idx[b*B + c]   for every (query i,
//                  slot s) that kept block b: queries that kept the same block
//                  are gathered (cp.async, one 16-byte piece per lane) as the
//                  128 rows of one MMA tile against that block's B keys, so
//                  each key block is read once per 128 queries instead of
//                  once per query.
// Integer-valued inputs make every product and partial sum an exact fp32
// integer, so the tensor-core results equal the sequential CPU sums.
//
// Warp roles of the persistent kernel: warp 0 TMA producer (the B tiles, and
// the A tiles of block scoring), warp 1 MMA issuer (+ TMEM owner), warps 2-5
// epilogue (TMEM -> keys -> global through a shared-memory staging tile),
// and for token scoring warps 6-9, which copy the gathered query rows. The
// TMEM accumulator is two deep, so the epilogue of one tile overlaps the MMAs
// of the next.
#include "kernels.cuh"
#include "tc.cuh"

namespace hsa {

__device__ int g_score_err;
__device__ int g_score_inject;  // test hook: short waits and one tile never produced

constexpr long long kInjectWaitCycles = 1ll << 21;  // about a millisecond

namespace {

using namespace tc;

HSA_DEV bool sg_wait(uint64_t* bar, uint32_t parity, bool& dead) {
  if (dead) return false;
  const long long lim = *(volatile int*)&g_score_inject ? kInjectWaitCycles : kWaitCycles;
  if (mbar_wait_bounded(bar, parity, &g_score_err, lim)) return true;
  dead = true;
  return false;
}
HSA_DEV bool sg_wait_warp(uint64_t* bar, uint32_t parity, bool& dead) {
  bool ok = false;
  if ((threadIdx.x & 31) == 0) ok = sg_wait(bar, parity, dead);
  ok = __shfl_sync(kFull, ok ? 1 : 0, 0) != 0;
  __syncwarp();
  dead = !ok;
  return ok;
}

template <int DK, int N, int NSPLIT>
struct SG {
  static constexpr int KB = DK / 64;                 // 128-byte column blocks per row
  static constexpr int A_BYTES = 128 * DK * 2;
  static constexpr int B_BYTES = NSPLIT * N * DK * 2;
  static constexpr int STAGE = A_BYTES + B_BYTES;
  static constexpr int NS = (200 * 1024) / STAGE > 4 ? 4 : (200 * 1024) / STAGE;
  static constexpr int SMEM = NS * STAGE + 1024;
  static constexpr int TMEM_COLS = 2 * N < 32 ? 32 : 2 * N;
};

// Tile source description shared by the roles.
struct TileArgs {
  // gathered mode (token scores)
  const int4* tiles;        // (block, first pair, pair count, -)
  const int* ntiles;        // device count of tiles
  const uint32_t* pairs;    // pair = row * m + slot
  int m, Bsz;
  const void* qsrc;         // gathered mode: q_idx rows [Lq][DK] bf16
  // tiled mode (block scores)
  int Lq, Lk, nb_tiles, m_tiles, nbc;
  // output
  uint32_t* out;
  int64_t ld;
};

// Tiled mode: does tile (mt, nt) hold any candidate block of any of its rows?
HSA_DEV bool block_tile_needed(const TileArgs& a, int mt, int nt, int N) {
  const int last_row = min(a.Lq - 1, mt * 128 + 127);
  const int64_t t_last = int64_t(a.Lk) - a.Lq + last_row;
  const int64_t nb_last = t_last / a.Bsz + 1;
  if (nb_last <= a.m) return false;            // every row keeps all its blocks
  return int64_t(nt) * N <= nb_last - 2;       // candidates are blocks 1 .. nb-2
}

// gathered mode: 4 more warps copy the query rows with cp.async
template <bool GATHER> constexpr int sg_threads() { return GATHER ? 320 : 192; }

template <int DK, int N, int NSPLIT, bool GATHER>
__global__ void __launch_bounds__(sg_threads<GATHER>(), 1) score_gemm_kernel(const __grid_constant__ CUtensorMap amap,
                                                            const __grid_constant__ CUtensorMap bmap,
                                                            TileArgs ta) {
  using C = SG<DK, N, NSPLIT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ __align__(8) uint64_t full[C::NS], empty[C::NS], tfull[2], tempty[2], done;
  __shared__ uint32_t tmem_base;
  __shared__ __align__(16) uint32_t stage[4][32 * 32];  // epilogue staging, one tile per warp
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    // gathered mode: the TMA bytes of B plus one arrival per query-row copying thread
    for (int s = 0; s < C::NS; ++s) { mbar_init(&full[s], GATHER ? 1 + 128 : 1); mbar_init(&empty[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull[b], 1); mbar_init(&tempty[b], 4); }
    mbar_init(&done, 1);
    fence_barrier_init();
  }
  if (warp == 1) { tmem_alloc(&tmem_base, C::TMEM_COLS); tmem_relinquish(); }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base;
  // the set-up above touches no global memory: under a programmatic
  // dependent launch it overlaps the previous kernel
  griddep_wait();
  griddep_launch();
  const int total = GATHER ? *ta.ntiles : ta.m_tiles * ta.nb_tiles;
  bool dead = false;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) { prefetch_tmap(&amap); prefetch_tmap(&bmap); }
    uint32_t it = 0;
    // a gathered tile's descriptor (its key block) is fetched one tile ahead
    int bn = (GATHER && blockIdx.x < total) ? ta.tiles[blockIdx.x].x : 0;
    for (int t = blockIdx.x; t < total && !dead; t += gridDim.x) {
      int a_row0 = 0, b_row0 = 0;
      if (GATHER) {
        b_row0 = bn * ta.Bsz;
        if (t + int(gridDim.x) < total) bn = ta.tiles[t + gridDim.x].x;
      } else {
        const int mt = t / ta.nb_tiles, nt = t % ta.nb_tiles;
        if (!block_tile_needed(ta, mt, nt, N)) continue;
        a_row0 = mt * 128;
        b_row0 = nt * N;
      }
      const int s = it % C::NS;
      if (!sg_wait_warp(&empty[s], ((it / C::NS) & 1) ^ 1, dead)) break;
      // test hook: CTA 0 never produces its first tile, so its consumer's wait runs out
      if (it == 0 && blockIdx.x == 0 && *(volatile int*)&g_score_inject) { ++it; continue; }
      uint8_t* a_s = sm + s * C::STAGE;
      uint8_t* b_s = a_s + C::A_BYTES;
      if (lane == 0) mbar_arrive_expect_tx(&full[s], GATHER ? C::B_BYTES : C::STAGE);
      __syncwarp();
      if (!GATHER && lane == 0) {
#pragma unroll
        for (int kb = 0; kb < C::KB; ++kb) tma_load_2d(a_s + kb * 128 * 128, &amap, &full[s], kb * 64, a_row0);
      }
      if (lane == 0) {
#pragma unroll
        for (int sp = 0; sp < NSPLIT; ++sp)
#pragma unroll
          for (int kb = 0; kb < C::KB; ++kb)
            tma_load_2d(b_s + sp * N * DK * 2 + kb * N * 128, &bmap, &full[s], kb * 64,
                        b_row0 + sp * ta.nbc);
      }
      ++it;
    }
    if (lane == 0) {  // drain armed loads
      bool d2 = false;
      for (uint32_t u = (it >= uint32_t(C::NS) ? it - C::NS : 0); u < it; ++u)
        sg_wait(&full[u % C::NS], (u / C::NS) & 1, d2);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, N, false, false);
      uint32_t it = 0;
      for (int t = blockIdx.x; t < total && !dead; t += gridDim.x) {
        if (!GATHER && !block_tile_needed(ta, t / ta.nb_tiles, t % ta.nb_tiles, N)) continue;
        const int s = it % C::NS, tb = it & 1;
        if (!sg_wait(&full[s], (it / C::NS) & 1, dead)) break;
        if (!sg_wait(&tempty[tb], ((it >> 1) & 1) ^ 1, dead)) break;
        tc_fence_after();
        if (GATHER) fence_proxy_async_smem();  // query rows landed by cp.async, read by the MMA
        const uint32_t a_s = smem_u32(sm + s * C::STAGE);
        const uint32_t b_s = a_s + C::A_BYTES;
        uint32_t acc = 0;
#pragma unroll
        for (int sp = 0; sp < NSPLIT; ++sp)
#pragma unroll
          for (int ks = 0; ks < DK / 16; ++ks) {
            const uint64_t a = smem_desc(a_s + (ks / 4) * 128 * 128 + (ks % 4) * 32, 16, 1024, kSw128);
            const uint64_t b = smem_desc(b_s + sp * N * DK * 2 + (ks / 4) * N * 128 + (ks % 4) * 32, 16, 1024, kSw128);
            mma_bf16(tmem + tb * N, a, b, idesc, acc);
            acc = 1;
          }
        mma_commit(&empty[s]);
        mma_commit(&tfull[tb]);
        ++it;
      }
      mma_commit(&done);
      bool d2 = false;
      sg_wait(&done, 0, d2);
    }
    __syncwarp();
  } else if (GATHER && warp >= 6) {
    // ------------------------------------------------------------ query-row copies
    // warp 6 + g copies rows 32g .. 32g+31 of each tile: lane l fetches the
    // query row of tile row 32g + l, the copying lanes take it by shuffle
    constexpr int CPR = DK / 8;          // 16-byte chunks per row
    constexpr int RPI = 32 / CPR;        // rows per warp instruction
    const int gw = warp - 6, c = lane % CPR, rsub = lane / CPR;
    const uint4* qb = reinterpret_cast<const uint4*>(ta.qsrc);
    uint32_t it = 0;
    // a tile's descriptor is fetched two tiles ahead, the query row one ahead
    const int g = int(gridDim.x);
    auto desc = [&](int tt) { return tt < total ? ta.tiles[tt] : make_int4(0, 0, 0, 0); };
    auto qrow_of = [&](const int4& d) -> int {
      const int r = 32 * gw + lane;
      return r < d.z ? int(ta.pairs[d.y + r] / uint32_t(ta.m)) : 0;
    };
    int qn = qrow_of(desc(blockIdx.x));
    int4 dn = desc(blockIdx.x + g);
    for (int t = blockIdx.x; t < total && !dead; t += gridDim.x) {
      const int qr = qn;
      qn = qrow_of(dn);
      dn = desc(t + 2 * g);
      const int s = it % C::NS;
      if (!sg_wait_warp(&empty[s], ((it / C::NS) & 1) ^ 1, dead)) break;
      const uint32_t a_s = smem_u32(sm + s * C::STAGE);
#pragma unroll
      for (int u = 0; u < 32 / RPI; ++u) {
        const int rr = u * RPI + rsub, row = 32 * gw + rr;
        const int q = __shfl_sync(kFull, qr, rr);
        cp_async16(a_s + (c >> 3) * (128 * 128) + row * 128 + (((c & 7) ^ (row & 7)) << 4),
                   qb + int64_t(q) * CPR + c);
      }
      cp_async_arrive(&full[s]);
      ++it;
    }
    cp_async_wait_all();  // every copy has landed before the CTA may exit
  } else {
    // ------------------------------------------------------------ epilogue
    // Each warp owns 32 accumulator rows (its TMEM lane quarter). Keys go out
    // 32 columns at a time through a 32 x 128-byte staging tile (16-byte
    // chunks XOR-swizzled by row), so that every global store instruction
    // writes four whole 128-byte row segments instead of 32 scattered pieces.
    const int quad = warp & 3, r = quad * 32 + lane;
    const uint32_t lane_addr = uint32_t(quad * 32) << 16;
    uint32_t* sb = stage[quad];
    const int rsub = lane >> 3, ch = lane & 7;
    uint32_t it = 0;
    // gathered mode: a tile's descriptor is fetched two tiles ahead and this
    // thread's pair one tile ahead, so neither load waits in the loop
    const int g = int(gridDim.x);
    auto desc = [&](int tt) { return tt < total ? ta.tiles[tt] : make_int4(0, 0, 0, 0); };
    auto pair_off = [&](const int4& d) { return r < d.z ? int64_t(ta.pairs[d.y + r]) * ta.ld : int64_t(-1); };
    int4 d_next = make_int4(0, 0, 0, 0);
    int64_t off_next = -1;
    if (GATHER) {
      off_next = pair_off(desc(blockIdx.x));
      d_next = desc(blockIdx.x + g);
    }
    for (int t = blockIdx.x; t < total && !dead; t += gridDim.x) {
      int64_t off = -1;  // element offset of this thread's row in out, or -1
      if (GATHER) {
        off = off_next;
        off_next = pair_off(d_next);
        d_next = desc(t + 2 * g);
      } else {
        const int mt = t / ta.nb_tiles, nt = t % ta.nb_tiles;
        if (!block_tile_needed(ta, mt, nt, N)) continue;
        const int row = mt * 128 + r;
        if (row < ta.Lq) off = int64_t(row) * ta.ld + int64_t(nt) * N;
      }
      // the rows this thread stores: 4 * i + rsub of the warp's 32
      int64_t roff[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) roff[i] = __shfl_sync(kFull, off, 4 * i + rsub);
      const int tb = it & 1;
      if (!sg_wait_warp(&tfull[tb], (it >> 1) & 1, dead)) break;
      tc_fence_after();
#pragma unroll 1
      for (int c0 = 0; c0 < N; c0 += 32) {
        float v[32];
        tmem_load_f32<32>(tmem + lane_addr + tb * N + c0, v);
        __syncwarp();  // the previous chunk has been read out of the staging tile
#pragma unroll
        for (int e = 0; e < 8; ++e)
          *reinterpret_cast<uint4*>(sb + lane * 32 + ((e ^ (lane & 7)) << 2)) =
              make_uint4(score_key(v[4 * e]), score_key(v[4 * e + 1]), score_key(v[4 * e + 2]),
                         score_key(v[4 * e + 3]));
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int rr = 4 * i + rsub;
          const uint4 x = *reinterpret_cast<const uint4*>(sb + rr * 32 + ((ch ^ (rr & 7)) << 2));
          if (roff[i] >= 0) *reinterpret_cast<uint4*>(ta.out + roff[i] + c0 + 4 * ch) = x;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[tb]);
      ++it;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
}

template <int DK, int N, int NSPLIT, bool GATHER>
bool launch_sg(const CUtensorMap& am, const CUtensorMap& bm, const TileArgs& ta, int grid, cudaStream_t s) {
  using C = SG<DK, N, NSPLIT>;
  auto kern = score_gemm_kernel<DK, N, NSPLIT, GATHER>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM) != cudaSuccess) return false;
  launch_kernel(true, kern, grid, sg_threads<GATHER>(), C::SMEM, s, am, bm, ta);
  count_launches(1);
  return true;
}

}  // namespace

// Block scores for rows [0, Lq): out[i][b] = key(q_idx[i] . ksum[b]) for the
// tiles that hold candidate blocks (others are left unwritten).
// bsplit: [3][nbc][d_idx] bf16 planes hi, mid, lo of ksum.
bool launch_block_score_gemm(const void* q_idx, const void* bsplit, int64_t Lq, int64_t Lk, int B, int m,
                             int d_idx, int64_t nbc, uint32_t* out, int64_t ld, cudaStream_t s) {
  constexpr int N = 64;
  CUtensorMap am, bm;
  if (!make_tmap_2d(&am, q_idx, uint64_t(Lq), uint64_t(d_idx), 128) ||
      !make_tmap_2d(&bm, bsplit, uint64_t(3 * nbc), uint64_t(d_idx), N))
    return false;
  TileArgs ta{};
  ta.m = m; ta.Bsz = B; ta.Lq = int(Lq); ta.Lk = int(Lk); ta.nbc = int(nbc);
  ta.m_tiles = int((Lq + 127) / 128);
  ta.nb_tiles = int((nbc + N - 1) / N);
  ta.out = out; ta.ld = ld;
  const int64_t tiles = int64_t(ta.m_tiles) * ta.nb_tiles;
  const int grid = int(tiles < num_sms() ? tiles : num_sms());
  if (grid == 0) return true;
  if (d_idx == 128) return launch_sg<128, N, 3, false>(am, bm, ta, grid, s);
  return launch_sg<64, N, 3, false>(am, bm, ta, grid, s);
}

// Token scores for the (row, slot) pairs listed per key block:
// out[pair][c] = key(q_idx[pair / m] . k_idx[block * B + c]), c < B.
bool launch_token_score_gemm(const void* q_idx, const void* k_idx, int64_t Lq, int64_t Lk, int B, int m,
                             int d_idx, const int4* tiles, const int* ntiles, const uint32_t* pairs,
                             int64_t max_tiles, uint32_t* out, cudaStream_t s) {
  // the query rows are copied by cp.async: only the key blocks go through a tensor map
  (void)Lq;
  CUtensorMap bm;
  if (!make_tmap_2d(&bm, k_idx, uint64_t(Lk), uint64_t(d_idx), B)) return false;
  const CUtensorMap& am = bm;
  TileArgs ta{};
  ta.tiles = tiles; ta.ntiles = ntiles; ta.pairs = pairs; ta.m = m; ta.Bsz = B; ta.qsrc = q_idx;
  ta.out = out; ta.ld = B;
  const int grid = int(max_tiles < num_sms() ? (max_tiles > 0 ? max_tiles : 1) : num_sms());
  if (d_idx == 128) {
    if (B == 128) return launch_sg<128, 128, 1, true>(am, bm, ta, grid, s);
    if (B == 64) return launch_sg<128, 64, 1, true>(am, bm, ta, grid, s);
    if (B == 256) return launch_sg<128, 256, 1, true>(am, bm, ta, grid, s);
  } else {
    if (B == 128) return launch_sg<64, 128, 1, true>(am, bm, ta, grid, s);
    if (B == 64) return launch_sg<64, 64, 1, true>(am, bm, ta, grid, s);
    if (B == 256) return launch_sg<64, 256, 1, true>(am, bm, ta, grid, s);
  }
  return false;
}

// Host side: turn the scoring kernels' test hook on or off on the current device.
bool score_set_inject(bool on) {
  const int v = on ? 1 : 0;
  return cudaMemcpyToSymbol(g_score_inject, &v, sizeof v) == cudaSuccess;
}

// Host side: whether a bounded wait of this kernel gave up on the current
// device since the flag was last cleared (synchronous copy; -1 on a CUDA error).
int score_wait_flag(bool reset) {
  int v = 0;
  if (cudaMemcpyFromSymbol(&v, g_score_err, sizeof v) != cudaSuccess) return -1;
  if (reset && v) {
    const int zero = 0;
    if (cudaMemcpyToSymbol(g_score_err, &zero, sizeof zero) != cudaSuccess) return -1;
  }
  return v != 0;
}

}  // namespace hsa
