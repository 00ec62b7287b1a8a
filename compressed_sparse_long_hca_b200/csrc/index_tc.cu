// Lightning-indexer scores on the 5th-generation tensor cores
// (csa_index_scores).
//
// Page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力": the query's index
// heads are scored against every compressed index key after a ReLU; podcast
// summary page, section "2.1 推理与计算效率": the indexer path runs in FP4.
//   s_j = sum_h w_h * max(0, q^_h . k^_j),   q^, k^ MXFP4 (E2M1, E8M0 per 32)
//
// Shape of the work: per query a [N x d_I] x [d_I x H_I] product with N up to
// 262,144 keys and H_I = 64, i.e. an FP4 GEMM whose A operand (the keys) is
// streamed once from HBM.  Each CTA owns a contiguous range of 128-key tiles
// (4 classic-cache blocks) of the flattened (query, tile) list:
//   * thread 0 streams each tile's codes and E8M0 scales from the paged cache
//     into a ring of shared-memory stages with bulk async copies (one per
//     block section; the cache stores codes in the no-swizzle K-major core
//     matrix order, so the copy lands ready for the MMA);
//   * the tile's key scales go to TMEM (tcgen05.st) and thread 0 issues the
//     block-scaled MMA  D[128 keys x 64 heads] = K^ Q^T  (kind::mxf4,
//     M=128, N=64, K=64 per instruction) into one of two TMEM accumulators;
//   * while the tensor core works on tile t, all four warps read tile t-1's
//     accumulator (one TMEM lane = one key, 64 columns = its 64 head dot
//     products) and reduce sum_h w_h max(0, d_h) in fixed head order.
// Every key's score is produced by the same instruction sequence whatever the
// grid, so launch variants and batch compositions return identical bits.
#include "common.cuh"
#include "tc.cuh"

namespace csa {

namespace {

constexpr int kStages = 6;
constexpr int kThreads = 128;
constexpr int kTileKeys = 128;
constexpr int kHeadsN = 64;            // MMA N (index heads, zero padded)
constexpr int kMaxCh = 4;              // d_I / 32 <= 4
// TMEM columns (allocation of 256)
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kAcc0 = 0, kAcc1 = 64, kSfa0 = 128, kSfa1 = 132, kSfb = 136;

struct IdxSmem {
  uint8_t codes[kStages][kTileKeys * kMaxCh * 16];   // 128 keys x up to 64 B, core-matrix order
  uint8_t sfs[kStages][kTileKeys * kMaxCh];          // per block: [32 keys][CH] bytes
  uint8_t qb[kHeadsN * kMaxCh * 16];                 // query codes, core-matrix order
  uint8_t sfq[kHeadsN][kMaxCh];
  float w[kHeadsN];
  uint64_t full[kStages];
  uint64_t mdone[2];
  uint32_t tmem_base;
  int abort;
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

// Number of 128-key tiles of query i (0 for an invalid query).
__device__ __forceinline__ int64_t query_tiles(const IndexTcArgs& a, int i, int64_t* n_keys, int* req_out) {
  const int req = a.req_ids[i];
  *req_out = req;
  if (req < 0 || req >= a.L.max_req) { *n_keys = 0; return 0; }
  const int64_t N = a.L.lengths()[(int64_t)a.layer * a.L.max_req + req] / kCsaM;
  *n_keys = N;
  if (N > a.ld) return 0;
  return (N + kTileKeys - 1) / kTileKeys;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 2) index_tc_kernel(IndexTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  IdxSmem& sm = *reinterpret_cast<IdxSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Layout& L = a.L;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int HI = L.HI, dI = L.dI, CH = dI / 32;
  const int CHs = (CH + 1) / 2 * 2;                 // chunks per key in smem (multiple of 2)
  const int n_mma = CHs / 2;                        // K = 64 per instruction
  const uint32_t sbo = (uint32_t)CHs * 128;

  // ---- per-query bookkeeping (every CTA computes the same prefix)
  if (blockIdx.x == 0) {
    for (int i = tid; i < a.n; i += kThreads) {
      int64_t N;
      int req;
      query_tiles(a, i, &N, &req);
      if (req < 0 || req >= L.max_req) { set_err(L, kErrBounds, i); a.n_valid[i] = 0; continue; }
      a.n_valid[i] = (int32_t)N;
      if (N > a.ld) set_err(L, kErrLd, i);
    }
  }
  int64_t total = 0;
  for (int i = 0; i < a.n; ++i) {
    int64_t N;
    int req;
    total += query_tiles(a, i, &N, &req);
  }
  const int64_t g0 = total * blockIdx.x / gridDim.x, g1 = total * (blockIdx.x + 1) / gridDim.x;
  if (g0 >= g1) return;

  // ---- set-up: TMEM, barriers, zero padding
  if (warp == 0) {
    tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) tc::mbar_init(&sm.full[s], 1);
    tc::mbar_init(&sm.mdone[0], 1);
    tc::mbar_init(&sm.mdone[1], 1);
    sm.abort = 0;
    tc::fence_mbar_init();
  }
  if (CHs != CH) {   // chunks past d_I stay zero for the whole kernel
    for (int x = tid; x < kStages * kTileKeys * kMaxCh * 16 / 16; x += kThreads)
      reinterpret_cast<uint4*>(&sm.codes[0][0])[x] = make_uint4(0, 0, 0, 0);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const uint32_t lane_base = (uint32_t)(warp * 32) << 16;

  // locate the first tile of this CTA
  int qi = 0;
  int64_t before = 0, Nq = 0;
  int req = 0;
  for (;; ++qi) {
    const int64_t t = query_tiles(a, qi, &Nq, &req);
    if (before + t > g0) break;
    before += t;
  }
  int64_t g = g0;
  uint32_t cnt = 0;                 // tiles processed by this CTA (barrier phases)
  bool ok = true;
  uint32_t pending = 0;             // thread 0: stages with a copy in flight
  uint32_t pend_par = 0;            //           and the parity that copy completes

  auto issue_load = [&](int stage, uint32_t gidx, int qry_req, int64_t tile, int64_t N) {
    const int32_t* bt = L.block_table(qry_req);
    uint32_t bytes = 0;
    for (int bb = 0; bb < 4; ++bb) {
      const int64_t lb = tile * 4 + bb;
      if (lb * kCsaPerBlock < N) bytes += 4u * (uint32_t)CH * 128u + 32u * (uint32_t)CH;
    }
    tc::mbar_arrive_expect_tx(&sm.full[stage], bytes);
    for (int bb = 0; bb < 4; ++bb) {
      const int64_t lb = tile * 4 + bb;
      if (lb * kCsaPerBlock >= N) continue;
      const char* bp = L.block(bt[lb], a.layer);
      uint8_t* dst = &sm.codes[stage][bb * 4 * CHs * 128];
      if (CHs == CH) {
        tc::bulk_g2s(dst, bp + L.blk_idx_codes, 4u * CH * 128u, &sm.full[stage]);
      } else {
        for (int rg = 0; rg < 4; ++rg)
          tc::bulk_g2s(dst + rg * CHs * 128, bp + L.blk_idx_codes + rg * CH * 128, (uint32_t)CH * 128u,
                       &sm.full[stage]);
      }
      tc::bulk_g2s(&sm.sfs[stage][bb * 32 * CH], bp + L.blk_idx_scale, 32u * CH, &sm.full[stage]);
    }
    pending |= 1u << stage;
    pend_par = (pend_par & ~(1u << stage)) | ((((gidx / kStages) & 1u)) << stage);
  };

  while (g < g1 && ok) {
    // ---- segment: tiles of query qi inside [g, g1)
    int64_t nt_q;
    while ((nt_q = query_tiles(a, qi, &Nq, &req)) == 0 || before + nt_q <= g) { before += nt_q; ++qi; }
    const int64_t t_first = g - before;
    const int64_t t_end = (g1 - before < nt_q) ? g1 - before : nt_q;
    const int64_t n_t = t_end - t_first;
    // quantise this query's index heads to MXFP4 in shared memory
    for (int x = tid; x < kHeadsN * CHs * 16 / 16; x += kThreads)
      reinterpret_cast<uint4*>(sm.qb)[x] = make_uint4(0, 0, 0, 0);
    __syncthreads();
    const float* q = a.q_idx + (int64_t)qi * HI * dI;
    for (int blk = warp; blk < HI * CH; blk += kThreads / 32) {
      const int h = blk / CH, c = blk % CH;
      const float x = q[h * dI + c * 32 + lane];
      float am = fabsf(x);
      for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
      const int e = mx_exponent(am);
      const float y = scale_pow2(x, e);
      const float y1 = __shfl_down_sync(0xffffffffu, y, 1);
      if ((lane & 1) == 0) sm.qb[(h >> 3) * sbo + c * 128 + (h & 7) * 16 + (lane >> 1)] = e2m1x2_rn(y, y1);
      if (lane == 0) sm.sfq[h][c] = (uint8_t)(e + 127);
    }
    for (int h = tid; h < kHeadsN; h += kThreads) sm.w[h] = h < HI ? a.w[(int64_t)qi * HI + h] : 0.f;
    __syncthreads();
    {
      uint32_t wq[2];
      for (int k = 0; k < 2; ++k) {
        const int h = lane + 32 * k;
        uint32_t word = 0;
        for (int c = 0; c < 4; ++c) word |= (uint32_t)((h < HI && c < CH) ? sm.sfq[h][c] : 127) << (8 * c);
        wq[k] = word;
      }
      tc::tmem_st_x2(tmem + lane_base + kSfb, wq[0], wq[1]);
      tc::tmem_wait_st();
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    if (tid == 0)
      for (int64_t p = 0; p < n_t && p < kStages; ++p)
        issue_load((int)((cnt + p) % kStages), cnt + (uint32_t)p, req, t_first + p, Nq);
    float* out = a.scores + (int64_t)qi * a.ld;
    // read tile `tile`'s accumulator (global tile counter gt) and store its scores
    auto epilogue = [&](uint32_t gt, int64_t tile) -> bool {
      const int b = gt & 1;
      if (!tc::mbar_wait(&sm.mdone[b], (gt >> 1) & 1)) return false;
      tc::tc_fence_after();
      uint32_t r[64];
      const uint32_t col = tmem + lane_base + (b ? kAcc1 : kAcc0);
      tc::tmem_ld_x16(col + 0, r);
      tc::tmem_ld_x16(col + 16, r + 16);
      tc::tmem_ld_x16(col + 32, r + 32);
      tc::tmem_ld_x16(col + 48, r + 48);
      tc::tmem_wait_ld();
      float s = 0.f;
#pragma unroll
      for (int h = 0; h < kHeadsN; ++h)
        if (h < HI) s = fmaf(sm.w[h], fmaxf(__uint_as_float(r[h]), 0.f), s);
      const int64_t j = tile * kTileKeys + warp * 32 + lane;
      if (j < Nq) out[j] = s;
      return true;
    };
    for (int64_t t = 0; t < n_t; ++t) {
      const uint32_t gt = cnt + (uint32_t)t;
      const int s = gt % kStages, b = gt & 1;
      const bool full_ok = tc::mbar_wait(&sm.full[s], (gt / kStages) & 1);
      if (full_ok) {
        if (tid == 0) pending &= ~(1u << s);
        // key scales of this tile -> TMEM (lane = key mod 32, column = key / 32)
        uint32_t wd[4];
        for (int m1 = 0; m1 < 4; ++m1) {
          const uint8_t* p = &sm.sfs[s][m1 * 32 * CH + lane * CH];
          uint32_t word = 0;
          for (int c = 0; c < 4; ++c) word |= (uint32_t)(c < CH ? p[c] : 127) << (8 * c);
          wd[m1] = word;
        }
        tc::tmem_st_x4(tmem + lane_base + (b ? kSfa1 : kSfa0), wd[0], wd[1], wd[2], wd[3]);
        tc::tmem_wait_st();
      }
      tc::tc_fence_before();
      ok = __syncthreads_and(ok && full_ok) != 0;
      tc::tc_fence_after();
      if (!ok) break;
      if (tid == 0) {
        const uint32_t a_base = tc::smem_u32(&sm.codes[s][0]);
        const uint32_t b_base = tc::smem_u32(sm.qb);
        for (int k = 0; k < n_mma; ++k) {
          const uint64_t ad = tc::smem_desc(a_base + k * 256, 128, sbo);
          const uint64_t bd = tc::smem_desc(b_base + k * 256, 128, sbo);
          const uint32_t id = tc::idesc_mxf4(128, kHeadsN, 2 * k, 2 * k);
          const uint32_t sfa = (tmem + (b ? kSfa1 : kSfa0)) | ((uint32_t)(2 * k) << 30);
          const uint32_t sfb = (tmem + kSfb) | ((uint32_t)(2 * k) << 30);
          tc::mma_mxf4(tmem + (b ? kAcc1 : kAcc0), ad, bd, id, sfa, sfb, k > 0 ? 1u : 0u);
        }
        tc::mma_commit(&sm.mdone[b]);
      }
      if (t > 0) {
        ok = epilogue(gt - 1, t_first + t - 1);
        // tile t-1's MMA has completed: its stage can take tile t-1+kStages
        if (ok && tid == 0 && t - 1 + kStages < n_t)
          issue_load((int)((gt - 1) % kStages), gt - 1 + kStages, req, t_first + t - 1 + kStages, Nq);
      }
    }
    if (ok) ok = epilogue(cnt + (uint32_t)n_t - 1, t_first + n_t - 1);
    cnt += (uint32_t)n_t;
    g += n_t;
    tc::tc_fence_before();
    ok = __syncthreads_and(ok) != 0;
    tc::tc_fence_after();
  }
  if (!ok) {
    if (tid == 0) {
      set_err(L, kErrTimeout, blockIdx.x);
      // let copies already in flight land before the shared memory goes away
      for (int s = 0; s < kStages; ++s)
        if (pending & (1u << s)) tc::mbar_wait(&sm.full[s], (pend_par >> s) & 1u, 200000000ull);
    }
    __syncthreads();
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, kTmemCols);
}

// Requesting ~100 KB keeps at most two CTAs on an SM, so that their two
// 256-column TMEM allocations always fit in the SM's 512 columns.
size_t index_tc_smem_bytes() {
  const size_t need = sizeof(IdxSmem) + 1024;
  return need > 100 * 1024 ? need : 100 * 1024;
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
  return cudaGetLastError();
}

}  // namespace csa
