// Lightning-indexer scores on the 5th-generation tensor cores
// (csa_index_scores).
//
// Page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力": the query's index
// heads are scored against every compressed index key after a ReLU; podcast
// summary page, section "2.1 推理与计算效率": the indexer path runs in FP4.
//   s_j = sum_h w_h * max(0, q^_h . k^_j),   q^, k^ MXFP4 (E2M1, E8M0 per 32)
//
// Shape of the work: per query an FP4 product [N keys x d_I] x [d_I x H_I]
// with N up to 262,144 and H_I = 64 whose A operand (the keys, 68 B each) is
// streamed once from HBM.  The cache stores the index keys of every 512-token
// page as one ready-made operand tile (codes in the no-swizzle K-major
// core-matrix order, scales in the 32 x 128-bit order of tcgen05.cp), so a
// 128-key tile is one bulk copy.  Two persistent CTAs per SM (their tcgen05
// issue latencies overlap) each own a contiguous range of tiles of the
// flattened (query, tile) list and run three roles:
//   * producer (warp 0): one bulk async copy per tile into a ring of
//     shared-memory stages;
//   * MMA (warp 1): one thread copies the tile's key scales into TMEM
//     (tcgen05.cp) and issues the block-scaled MMA
//     D[128 keys x 64 heads] = K^ Q^T (kind::mxf4, M=128, N=64, K=64 per
//     instruction) into one of four TMEM accumulators;
//   * epilogue (warps 2-9, two groups of four warps taking alternate tiles):
//     read a finished accumulator (one TMEM lane = one key, 64 columns = its
//     64 head dot products) and reduce sum_h w_h max(0, d_h) in a fixed
//     order.  At a query boundary they quantise the next query's index heads
//     to MXFP4 (the B operand and its scale chunk).
// Every key's score comes from the same instruction sequence whatever the
// grid, so launch variants and batch compositions return identical bits.
// All waits are bounded: a stuck pipeline records a timeout in the device
// error word, lets in-flight copies land, frees TMEM and returns.
#include "common.cuh"
#include "tc.cuh"

namespace csa {

namespace {

constexpr int kStages = 8;             // shared-memory stages of key tiles
constexpr int kNA = 3;                 // TMEM accumulators (and key-scale buffers)
constexpr int kEpiGroups = 2;          // epilogue groups, alternate tiles
constexpr int kGroupThreads = 128;     // one thread per key of a tile
constexpr int kEpiThreads = kEpiGroups * kGroupThreads;
constexpr int kThreads = 64 + kEpiThreads;   // warp 0 producer, warp 1 MMA, warps 2-9 epilogue
constexpr int kCtasPerSm = 2;          // two CTAs per SM overlap their issue latencies
constexpr int kHeadsN = 64;            // MMA N (index heads, zero padded)
constexpr int kMaxCh = 4;              // d_I / 32 <= 4
constexpr int kTileBytes = kCsaPerPage * kMaxCh * 16 + kSfChunk;   // codes + scale chunk
constexpr int kPassTiles = 128;        // tiles per pass (page-table window in smem)
constexpr int kMaxSeg = 64;            // queries per pass
constexpr int kMaxQ = 256;             // queries whose tile counts are kept in shared memory
constexpr uint32_t kTmemCols = 256;    // per CTA; two CTAs fill the SM's 512 columns
constexpr uint32_t kSfaCol = 192;      // + 4 * accumulator index
constexpr uint32_t kSfbCol = 204;

struct IdxSmem {
  uint8_t tiles[kStages][kTileBytes];                // one page's index tile per stage
  uint8_t qb[kHeadsN * kMaxCh * 16];                 // query codes, core-matrix order
  uint8_t qsf[kSfChunk];                             // query scales, tcgen05.cp order
  alignas(16) float w[kHeadsN];
  int32_t pgs[kPassTiles];                           // pool page of every tile of the pass
  // segments of the pass: one per query touched
  int32_t seg_q[kMaxSeg];
  int32_t seg_n[kMaxSeg];
  int64_t seg_t0[kMaxSeg];
  int64_t seg_N[kMaxSeg];
  int32_t n_seg;
  int32_t q_tiles[kMaxQ];                            // tiles of query i (i < kMaxQ)
  int64_t q_N[kMaxQ];                                // keys of query i
  int64_t red[kThreads / 32];
  uint64_t full[kStages], stage_empty[kStages];
  uint64_t acc_full[kNA], acc_empty[kNA];
  uint64_t q_ready;
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort;
};

struct IndexTcArgs {
  Layout L;
  int layer;
  int n;
  const int32_t* req_ids;
  const float* q_idx;
  const float* w;
  float* scores;
  int64_t ld;
  int32_t* n_valid;
};

// Number of 128-key tiles of query i (0 for an invalid query); N = its keys.
__device__ __forceinline__ int64_t query_tiles(const IndexTcArgs& a, int i, int64_t* n_keys, int* req_out) {
  const int req = a.req_ids[i];
  *req_out = req;
  if (req < 0 || req >= a.L.max_req) { *n_keys = 0; return 0; }
  const int64_t N = a.L.lengths()[(int64_t)a.layer * a.L.max_req + req] / kCsaM;
  *n_keys = N;
  if (N > a.ld) return 0;
  return (N + kCsaPerPage - 1) / kCsaPerPage;
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_or_abort(IdxSmem& sm, uint64_t* bar, uint32_t parity) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = tc::globaltimer_ns();
  for (uint32_t spin = 0;; ++spin) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    if ((spin & 127u) == 127u) {
      if (sm.abort) return false;
      if (tc::globaltimer_ns() - t0 > 2000000000ull) { sm.abort = 1; return false; }
    }
  }
}

}  // namespace

__global__ void __launch_bounds__(kThreads, kCtasPerSm) index_tc_kernel(IndexTcArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  IdxSmem& sm = *reinterpret_cast<IdxSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const Layout& L = a.L;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int HI = L.HI, dI = L.dI, CH = dI / 32, CHs = L.CHs;
  const int n_mma = CHs / 2;                        // K = 64 per instruction
  const uint32_t sbo = (uint32_t)CHs * 128;
  const uint32_t tile_bytes = (uint32_t)L.idx_tile_bytes;
  const uint32_t sf_off = (uint32_t)(kCsaPerPage * CHs * 16);

  // ---- set-up (overlaps the bookkeeping's global loads below)
  if (warp == 1) {
    tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) { tc::mbar_init(&sm.full[s], 1); tc::mbar_init(&sm.stage_empty[s], 1); }
    for (int k = 0; k < kNA; ++k) { tc::mbar_init(&sm.acc_full[k], 1); tc::mbar_init(&sm.acc_empty[k], kGroupThreads); }
    tc::mbar_init(&sm.q_ready, 1);
    tc::mbar_init(&sm.drain, 1);
    sm.abort = 0;
    tc::fence_mbar_init();
  }

  // ---- per-query bookkeeping (one thread per query); every CTA computes
  //      the same tile total
  int64_t total = 0;
  {
    int64_t part = 0;
    for (int i = tid; i < a.n; i += kThreads) {
      int64_t N;
      int req;
      const int64_t nt = query_tiles(a, i, &N, &req);
      if (i < kMaxQ) { sm.q_tiles[i] = (int32_t)nt; sm.q_N[i] = N; }
      part += nt;
      if (blockIdx.x == 0) {
        if (req < 0 || req >= L.max_req) { set_err(L, kErrBounds, i); a.n_valid[i] = 0; continue; }
        a.n_valid[i] = (int32_t)N;
        if (N > a.ld) set_err(L, kErrLd, i);
      }
    }
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) sm.red[warp] = part;
    tc::tc_fence_before();
    __syncthreads();                       // also publishes the TMEM address and the barriers
    tc::tc_fence_after();
    for (int w = 0; w < kThreads / 32; ++w) total += sm.red[w];
  }
  const uint32_t tmem = sm.tmem_base;
  const int64_t g0 = total * blockIdx.x / gridDim.x, g1 = total * (blockIdx.x + 1) / gridDim.x;
  if (g0 >= g1) {                          // no tiles for this CTA: nothing was issued
    if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);
    return;
  }

  // role state (each role only uses its own)
  uint32_t u_base = 0;       // CTA-wide tile counter at the start of the pass (barrier phases)
  uint32_t seg_count = 0;    // segments processed (q_ready phases)
  uint32_t last_issue[kStages];
  for (int s = 0; s < kStages; ++s) last_issue[s] = 0xFFFFFFFFu;
  int qi = 0;
  int64_t before = 0;        // tiles of queries < qi
  int64_t g = g0;

  while (g < g1 && !sm.abort) {
    // ---- pass prologue: segment table and page window (all threads)
    __syncthreads();
    if (tid == 0) {
      int ns = 0;
      int64_t gg = g, used = 0;
      while (gg < g1 && used < kPassTiles && ns < kMaxSeg) {
        int64_t N, nt;
        if (qi < kMaxQ) {
          nt = sm.q_tiles[qi];
          N = sm.q_N[qi];
        } else {
          int req;
          nt = query_tiles(a, qi, &N, &req);
        }
        if (nt == 0 || before + nt <= gg) { before += nt; ++qi; continue; }
        const int64_t t0 = gg - before;
        int64_t cnt = (g1 - before < nt ? g1 - before : nt) - t0;
        if (cnt > kPassTiles - used) cnt = kPassTiles - used;
        sm.seg_q[ns] = qi;
        sm.seg_t0[ns] = t0;
        sm.seg_n[ns] = (int32_t)cnt;
        sm.seg_N[ns] = N;
        ++ns;
        used += cnt;
        gg += cnt;
      }
      sm.n_seg = ns;
    }
    __syncthreads();
    {
      int base = 0;
      for (int sg = 0; sg < sm.n_seg; ++sg) {
        const int32_t* pt = L.page_table(a.req_ids[sm.seg_q[sg]]);
        for (int x = tid; x < sm.seg_n[sg]; x += kThreads) sm.pgs[base + x] = pt[sm.seg_t0[sg] + x];
        base += sm.seg_n[sg];
      }
    }
    __syncthreads();
    const int n_seg = sm.n_seg;
    int pass_tiles = 0;
    for (int sg = 0; sg < n_seg; ++sg) pass_tiles += sm.seg_n[sg];

    if (warp == 0) {
      // ================= producer: one bulk copy per tile =================
      // The whole warp walks the loop; one elected lane issues.
      for (int k = 0; k < pass_tiles; ++k) {
        const uint32_t u = u_base + (uint32_t)k;
        const int s = u % kStages;
        const bool ok = u < (uint32_t)kStages || wait_or_abort(sm, &sm.stage_empty[s], ((u / kStages) - 1) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        const char* src = L.page(sm.pgs[k], a.layer) + L.pg_idx_codes;
        if (tc::elect_one()) {
          tc::mbar_arrive_expect_tx(&sm.full[s], tile_bytes);
          tc::bulk_g2s(&sm.tiles[s][0], src, tile_bytes, &sm.full[s]);
        }
        __syncwarp();
        last_issue[s] = u;
      }
    } else if (warp == 1) {
      // ================= MMA issuer =================
      // The whole warp walks the loop; one elected lane issues the tcgen05
      // operations, whose operands are warp-uniform.
      uint32_t u = u_base;
      bool ok = true;
      for (int sg = 0; sg < n_seg && ok; ++sg) {
        ok = wait_or_abort(sm, &sm.q_ready, seg_count & 1);
        ++seg_count;
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc::tc_fence_after();
        if (tc::elect_one()) tc::tmem_cp_32x128b_x4(tmem + kSfbCol, tc::smem_desc(tc::smem_u32(sm.qsf), 128, 128));
        __syncwarp();
        const int nt = sm.seg_n[sg];
        for (int k = 0; k < nt; ++k, ++u) {
          const int s = u % kStages, na = u % kNA;
          ok = wait_or_abort(sm, &sm.full[s], (u / kStages) & 1) &&
               (u < (uint32_t)kNA || wait_or_abort(sm, &sm.acc_empty[na], ((u / kNA) - 1) & 1));
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t a_base = tc::smem_u32(&sm.tiles[s][0]);
          const uint32_t b_base = tc::smem_u32(sm.qb);
          const uint32_t sfa_col = tmem + kSfaCol + 4 * na;
          if (tc::elect_one()) {
            tc::tmem_cp_32x128b_x4(sfa_col, tc::smem_desc(a_base + sf_off, 128, 128));
            for (int m = 0; m < n_mma; ++m) {
              const uint64_t ad = tc::smem_desc(a_base + m * 256, 128, sbo);
              const uint64_t bd = tc::smem_desc(b_base + m * 256, 128, sbo);
              const uint32_t id = tc::idesc_mxf4(128, kHeadsN, 2 * m, 2 * m);
              tc::mma_mxf4(tmem + 64 * na, ad, bd, id, sfa_col | ((uint32_t)(2 * m) << 30),
                           (tmem + kSfbCol) | ((uint32_t)(2 * m) << 30), m > 0 ? 1u : 0u);
            }
            tc::mma_commit(&sm.acc_full[na]);
            tc::mma_commit(&sm.stage_empty[s]);
          }
          __syncwarp();
        }
      }
    } else {
      // ================= epilogue warps =================
      const int et = tid - 64;                       // 0 .. kEpiThreads-1
      const int grp = et / kGroupThreads;            // this group takes tiles u with u % kEpiGroups == grp
      const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
      const int key_in_tile = (warp & 3) * 32 + lane;
      uint32_t u = u_base;
      bool ok = true;
      // Every epilogue thread walks all segments and reaches every named
      // barrier, also after an abort (the work is then skipped), so that no
      // thread can be left waiting at a barrier another thread has left.
      for (int sg = 0; sg < n_seg; ++sg) {
        const int qq = sm.seg_q[sg];
        const int nt = sm.seg_n[sg];
        const int64_t t0 = sm.seg_t0[sg], N = sm.seg_N[sg];
        // -- all tiles of earlier segments are finished: every MMA that read
        //    the previous query's operands has completed.  Quantise this
        //    query's index heads: B operand codes and its scale chunk.
        tc::named_bar_sync(1, kEpiThreads);
        for (int x = et; x < kHeadsN * CHs; x += kEpiThreads)
          reinterpret_cast<uint4*>(sm.qb)[x] = make_uint4(0, 0, 0, 0);
        for (int x = et; x < kSfChunk / 4; x += kEpiThreads)
          reinterpret_cast<uint32_t*>(sm.qsf)[x] = 0x7F7F7F7Fu;        // scale 1.0 for padding
        tc::named_bar_sync(1, kEpiThreads);
        const float* q = a.q_idx + (int64_t)qq * HI * dI;
        for (int blk = et; blk < HI * CH; blk += kEpiThreads) {
          const int h = blk / CH, c = blk % CH;
          const float4* src = reinterpret_cast<const float4*>(q + h * dI + c * 32);
          float v[32];
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const float4 f = src[x];
            v[4 * x] = f.x; v[4 * x + 1] = f.y; v[4 * x + 2] = f.z; v[4 * x + 3] = f.w;
          }
          float am = 0.f;
#pragma unroll
          for (int x = 0; x < 32; ++x) am = fmaxf(am, fabsf(v[x]));
          const int e = mx_exponent(am);
          uint32_t pk[4] = {0, 0, 0, 0};
#pragma unroll
          for (int x = 0; x < 16; ++x)
            pk[x >> 2] |= (uint32_t)e2m1x2_rn(scale_pow2(v[2 * x], e), scale_pow2(v[2 * x + 1], e)) << (8 * (x & 3));
          *reinterpret_cast<uint4*>(&sm.qb[(h >> 3) * sbo + c * 128 + (h & 7) * 16]) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
          sm.qsf[Layout::idx_sf_off(h, c)] = (uint8_t)(e + 127);
        }
        for (int h = et; h < kHeadsN; h += kEpiThreads) sm.w[h] = h < HI ? a.w[(int64_t)qq * HI + h] : 0.f;
        tc::fence_proxy_async_smem();
        tc::named_bar_sync(1, kEpiThreads);
        if (et == 0) tc::mbar_arrive(&sm.q_ready);
        float* out = a.scores + (int64_t)qq * a.ld;
        for (int k = (int)((grp + kEpiGroups - (int)(u % kEpiGroups)) % kEpiGroups); k < nt && ok;
             k += kEpiGroups) {
          const uint32_t uk = u + (uint32_t)k;
          const int na = uk % kNA;
          if (!(ok = wait_or_abort(sm, &sm.acc_full[na], (uk / kNA) & 1))) break;
          tc::tc_fence_after();
          // two halves of 32 head columns (fewer live registers); four
          // interleaved partial sums (heads h = 4i + p), combined in a fixed order
          const uint32_t col = tmem + lane_base + 64 * na;
          const float4* w4 = reinterpret_cast<const float4*>(sm.w);
          float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t r[32];
            tc::tmem_ld_x16(col + 32 * half, r);
            tc::tmem_ld_x16(col + 32 * half + 16, r + 16);
            tc::tmem_wait_ld();
            if (half == 1) {
              tc::tc_fence_before();
              tc::mbar_arrive(&sm.acc_empty[na]);
            }
#pragma unroll
            for (int h4 = 0; h4 < 8; ++h4) {
              if (32 * half + h4 * 4 < HI) {
                const float4 wv = w4[8 * half + h4];
                p0 = fmaf(wv.x, fmaxf(__uint_as_float(r[4 * h4 + 0]), 0.f), p0);
                p1 = fmaf(wv.y, fmaxf(__uint_as_float(r[4 * h4 + 1]), 0.f), p1);
                p2 = fmaf(wv.z, fmaxf(__uint_as_float(r[4 * h4 + 2]), 0.f), p2);
                p3 = fmaf(wv.w, fmaxf(__uint_as_float(r[4 * h4 + 3]), 0.f), p3);
              }
            }
          }
          const int64_t j = (t0 + k) * kCsaPerPage + key_in_tile;
          if (j < N) out[j] = (p0 + p1) + (p2 + p3);
        }
        u += (uint32_t)nt;
        if (!ok) sm.abort = 1;
      }
    }
    u_base += (uint32_t)pass_tiles;
    g += pass_tiles;
    __syncthreads();
  }
  if (warp == 1 && u_base > 0) {
    // every tcgen05 operation this CTA issued has finished before TMEM is released
    if (tc::elect_one()) tc::mma_commit(&sm.drain);
    __syncwarp();
    tc::mbar_wait(&sm.drain, 0, 200000000ull);
  }
  if (sm.abort) {
    if (tid == 0) {
      set_err(L, kErrTimeout, blockIdx.x);
      // let copies already in flight land before the shared memory goes away
      for (int s = 0; s < kStages; ++s)
        if (last_issue[s] != 0xFFFFFFFFu) tc::mbar_wait(&sm.full[s], (last_issue[s] / kStages) & 1, 200000000ull);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);
}

// Sized so that exactly two CTAs share an SM (at most 113 KB each): their
// two 256-column TMEM allocations then always fit the SM's 512 columns.
size_t index_tc_smem_bytes() {
  const size_t need = sizeof(IdxSmem) + 128;
  return need > 80 * 1024 ? need : 80 * 1024;
}

cudaError_t launch_index_tc(const Layout& L, int layer, int n, const int32_t* req_ids, const float* q_idx,
                            const float* w, float* scores, int64_t ld, int32_t* n_valid, int ctas,
                            cudaStream_t st) {
  static bool attr = false;
  if (!attr) {
    cudaError_t e = cudaFuncSetAttribute(index_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)index_tc_smem_bytes());
    if (e != cudaSuccess) return e;
    attr = true;
  }
  IndexTcArgs a{L, layer, n, req_ids, q_idx, w, scores, ld, n_valid};
  index_tc_kernel<<<ctas, kThreads, index_tc_smem_bytes(), st>>>(a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace csa
