// Multi-query decode attention on the 5th-generation tensor cores
// (csa_hca_decode_attn).
//
// Page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力": the selected
// compressed entries and the sliding window's raw tokens are fed together to
// multi-query attention (all query heads share one KV head); section
// "HCA——重度压缩注意力": HCA attends densely to every compressed entry, both
// keep the latest 128 raw tokens, each head has a learnable sink logit added
// to the softmax denominator, RoPE acts on the last 64 dims only, and the
// stored KV is FP8 (non-RoPE dims) + BF16 (RoPE dims).
//
// Rows of a query: the entries of its top-k list in list order (HCA: every
// completed entry), then the window in ascending position; a -1 in the list
// is an empty row.  K = V = the stored row.  Because the KV head is shared,
// QK^T and PV are dense products.
//
// Reduction order (fixed by the query alone).  The rows are cut into tiles
// of 128.  Each tile gives a partial result
//     m_t = max_r u_r,  l_t = sum_r e^{u_r - m_t},  O_t = sum_r e^{u_r - m_t} V_r
// and the partials are folded in tile order,
//     m' = max(m, m_t),  l' = l e^{m-m'} + l_t e^{m_t-m'},  O' = O e^{m-m'} + O_t e^{m_t-m'};
// the sink enters last: out = O e^{m-mu} / (l e^{m-mu} + e^{sink-mu}),
// mu = max(m, sink).  Page "DeepSeek不惜代价保住它！V4关键特性被挖出来了",
// section "牺牲了什么" (and page "DeepSeek V4 底层逻辑全解析：从 V3 到 V4，真正
// 升级了什么？", section "升级点 3"): the authors give up split-KV because its
// reduction path changes with the batch, and ship two attention kernels (for
// a well-fed and an under-fed GPU) that agree bit for bit.  Here both launch variants
// compute the same tiles with the same code and fold them with the same
// arithmetic:
//   * whole-query launch (well-fed GPU): one CTA per (query, head group)
//     walks the tiles and folds each into a running accumulator in TMEM;
//   * split launch (under-fed GPU): one CTA per (query, head group, tile)
//     writes its partial to the caller's workspace, and attn_fold_kernel
//     folds them in tile order, one thread per output element.
// Nothing in either path depends on the batch.
//
// Per tile, in a CTA of 8 warps:
//   * the rows' addresses are resolved (page table, ring slot) into shared
//     memory; all threads then gather the rows, 8 rows x 4 16-byte chunks per
//     warp instruction, dequantise the FP8 codes exactly to BF16 and store
//     them in the no-swizzle core-matrix order (the first tile is gathered by
//     warps 0-3 alone, while warps 4-7 prepare the query heads);
//   * QK: S^T[128 rows x G heads] = K_tile Q^T (kind::f16, M = 128 rows,
//     N = G heads) into TMEM, in two accumulators: the FP8 dims (scaled by
//     the row's FP8 scale afterwards) and the BF16 RoPE dims;
//   * softmax statistics of the tile: one thread per (row, 16 heads);
//   * PV: O_t^T[dims x G] = V^T P^T, P^T in BF16; the FP8 dims use
//     (P * row scale)^T, the RoPE dims P^T, each into its own accumulator.
#include <cooperative_groups.h>

#include <mutex>
#include <vector>

#include "attn_common.cuh"
#include "common.cuh"
#include "tc.cuh"

namespace csa {

namespace {

constexpr int kAttThreads = 256;
constexpr int kMaxLoads = 18;      // 16-byte loads per thread per tile (D <= 512)

constexpr int kPgtCache = 2048;    // page-table entries of the query's request kept in shared memory (1M tokens)

struct AttnSmem {
  int Dp;             // head dim padded to a multiple of 128
  int64_t tile, qs, pt, rowf8, rowbf, rsc, stats, pgt, bars, total;
};

__host__ __device__ inline AttnSmem attn_smem(int D, int G) {
  AttnSmem s{};
  s.Dp = (D + 127) / 128 * 128;
  int64_t o = 0;
  s.tile = o;  o += (int64_t)kTileRows * s.Dp * 2;           // BF16 rows, core-matrix order
  s.qs = o;    o += (int64_t)G * s.Dp * 2;                   // BF16 query heads
  s.pt = o;    o += (int64_t)kTileRows * G * 2 * 2;          // BF16 P^T and (P*scale)^T (before the first tile:
                                                             // cos / sin of the RoPE pairs; after the last: the
                                                             // cluster fold's (m, l) of every chunk)
  s.rowf8 = o; o += (int64_t)kTileRows * 8;                  // row addresses (FP8 part)
  s.rowbf = o; o += (int64_t)kTileRows * 8;                  // row addresses (BF16 part)
  s.rsc = o;   o += (int64_t)kTileRows * 4;                  // row FP8 scales
  s.stats = o; o += (int64_t)14 * 32 * 4;
  s.pgt = o;   o += (int64_t)kPgtCache * 4;                  // page table of the request (first entries)
  o = (o + 15) / 16 * 16;
  s.bars = o;  o += 64;
  s.total = o;
  return s;
}

__device__ __forceinline__ uint4 ld_nc16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "l"(p));
  return v;
}

// Reduction over the 32 lanes of a warp of 16 values per lane (lane = row,
// value e = head e), by exchanging halves: 16 shuffles.  Lane l returns the
// reduction for head l >> 1 (lanes 2h and 2h+1 hold the same value).  The
// order of the operations is fixed.
template <bool kMax>
__device__ __forceinline__ float warp_reduce16(const float (&v)[16], int lane) {
  auto op = [](float x, float y) { return kMax ? fmaxf(x, y) : x + y; };
  float a8[8], a4[4], a2[2];
  const bool u16 = lane & 16, u8 = lane & 8, u4 = lane & 4, u2 = lane & 2;
#pragma unroll
  for (int j = 0; j < 8; ++j)
    a8[j] = op(u16 ? v[8 + j] : v[j], __shfl_xor_sync(0xffffffffu, u16 ? v[j] : v[8 + j], 16));
#pragma unroll
  for (int j = 0; j < 4; ++j)
    a4[j] = op(u8 ? a8[4 + j] : a8[j], __shfl_xor_sync(0xffffffffu, u8 ? a8[j] : a8[4 + j], 8));
#pragma unroll
  for (int j = 0; j < 2; ++j)
    a2[j] = op(u4 ? a4[2 + j] : a4[j], __shfl_xor_sync(0xffffffffu, u4 ? a4[j] : a4[2 + j], 4));
  const float a1 = op(u2 ? a2[1] : a2[0], __shfl_xor_sync(0xffffffffu, u2 ? a2[0] : a2[1], 2));
  return op(a1, __shfl_xor_sync(0xffffffffu, a1, 1));
}

// Address of row `r` of tile `tt` and of its FP8 scale (*scp, null for no
// row; the scale is loaded with the row's gather, off the address chain);
// returns whether the row exists.  The first n_pgt page-table entries of the
// request are read from `pgt` (shared memory), the others from the arena.
__device__ __forceinline__ bool resolve_row(const AttnArgs& a, const QueryGeom& g, int i, int tt, int r,
                                            uint64_t* rowf8, uint64_t* rowbf, const float** scp, const int32_t* pgt,
                                            int n_pgt) {
  const Layout& L = a.L;
  const int64_t rr = (int64_t)tt * kTileRows + r;
  const uint8_t* f8 = nullptr;
  const uint16_t* bf = nullptr;
  const float* sc = nullptr;
  if (rr < g.n_list) {
    int64_t j = g.csa ? (int64_t)a.topk[(int64_t)i * a.k + rr] : rr;
    if (j >= g.n_entries) {
      set_err(L, kErrBounds, 2000000 + i);
      j = -1;
    }
    if (j >= 0) {
      const int P = L.rows_per_page(a.layer);
      const int64_t pi = j / P;
      const int s = (int)(j % P);
      const char* pp = L.page(pi < n_pgt ? pgt[pi] : L.page_table(g.req)[pi], a.layer);
      f8 = reinterpret_cast<const uint8_t*>(pp) + (int64_t)s * L.kv_fp8_bytes;
      bf = reinterpret_cast<const uint16_t*>(pp + (g.csa ? L.pg_csa_bf16 : L.pg_hca_bf16)) + (int64_t)s * L.R;
      sc = reinterpret_cast<const float*>(pp + (g.csa ? L.pg_csa_scale : L.pg_hca_scale)) + s;
    }
  } else if (rr < g.total) {
    const int64_t p = g.w0 + (rr - g.n_list);
    const char* st = ring_base(a, g, p);
    const int slot = (int)(p % kWindow);
    f8 = reinterpret_cast<const uint8_t*>(st + L.ring_fp8) + (int64_t)slot * (L.D - L.R);
    bf = reinterpret_cast<const uint16_t*>(st + L.ring_bf16) + (int64_t)slot * L.R;
    sc = reinterpret_cast<const float*>(st + L.ring_scale) + slot;
  }
  rowf8[r] = reinterpret_cast<uint64_t>(f8);
  rowbf[r] = reinterpret_cast<uint64_t>(bf);
  *scp = sc;
  return f8 != nullptr;
}

constexpr int kClusterFoldMax = 16;    // chunks per query the cluster fold serves (cluster size)

// Split launch with the fold in the cluster.  The CTAs of one (query, head
// group), one per chunk, form a thread-block cluster; each has staged its
// chunk's (m_c, l_c) per head and O_c [G][D] in its own shared memory (an
// empty chunk: m_c = -inf).  After a cluster barrier every CTA folds a slice
// of the head group's outputs, reading the chunks' partials from the other
// CTAs' shared memory in chunk order, with the arithmetic of
// attn_fold_kernel, so the bits are the same as the workspace path's.  A
// second cluster barrier keeps every CTA's shared memory alive until all
// reads of it are done.
__device__ __noinline__ void cluster_fold(int G, int H, int D, const float* sink, uint16_t* out, int n_chunks, int i,
                                          int h0, const float* o_stage, const float2* ml_stage, float2* ml_all) {
  namespace cg = cooperative_groups;
  cg::cluster_group cl = cg::this_cluster();
  const int C = (int)cl.num_blocks();
  const int rank = (int)cl.block_rank();
  const int nch = n_chunks < C ? n_chunks : C;
  cl.sync();
  for (int x = threadIdx.x; x < nch * G; x += blockDim.x)
    ml_all[x] = *cl.map_shared_rank(ml_stage + x % G, (unsigned)(x / G));
  __syncthreads();
  tc::griddep_wait();          // (a CTA without rows has not waited yet) nothing is written before
  const int n4 = G * D / 4;
  const int per = (n4 + C - 1) / C;
  const int u_end = (rank + 1) * per < n4 ? (rank + 1) * per : n4;
  for (int u = rank * per + (int)threadIdx.x; u < u_end; u += blockDim.x) {
    const int hh = (4 * u) / D, d = (4 * u) % D;
    const int h = h0 + hh;
    if (h >= H) continue;
    float4 v[kClusterFoldMax];
#pragma unroll
    for (int c = 0; c < kClusterFoldMax; ++c)
      if (c < nch) v[c] = *reinterpret_cast<const float4*>(cl.map_shared_rank(o_stage + hh * D + d, (unsigned)c));
    float m = -INFINITY, l = 0.f;
    float o[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int c = 0; c < kClusterFoldMax; ++c) {
      if (c >= nch) break;
      const float2 ml = ml_all[c * G + hh];
      if (ml.x == -INFINITY) continue;
      float mn, al, be;
      fold_coef(m, ml.x, mn, al, be);
      l = fold_val(l, al, ml.y, be);
      o[0] = fold_val(o[0], al, v[c].x, be);
      o[1] = fold_val(o[1], al, v[c].y, be);
      o[2] = fold_val(o[2], al, v[c].z, be);
      o[3] = fold_val(o[3], al, v[c].w, be);
      m = mn;
    }
    float cm, dn;
    finish_coef(m, sink[h], l, cm, dn);
    uint2 pk;
    pk.x = (uint32_t)finish_val(o[0], cm, dn) | ((uint32_t)finish_val(o[1], cm, dn) << 16);
    pk.y = (uint32_t)finish_val(o[2], cm, dn) | ((uint32_t)finish_val(o[3], cm, dn) << 16);
    *reinterpret_cast<uint2*>(out + ((int64_t)i * H + h) * D + d) = pk;
  }
  cl.sync();
}

}  // namespace

// Both launch variants.  kSplit: grid (chunks_max, head groups, n), one chunk
// of tiles per CTA, its partial to the workspace.  Otherwise grid (n, head
// groups): the CTA walks every tile, folding the tiles of a chunk into a
// chunk result and (chunks of more than one tile) the chunk results into a
// total.
template <bool kSplit>
__global__ void __launch_bounds__(kAttThreads, 1) attn_tc_kernel(AttnArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Layout& L = a.L;
  const int D = L.D, R = L.R, H = L.H, G = a.G;
  const AttnSmem S = attn_smem(D, G);
  const int Dp = S.Dp;
  const uint32_t sbo_rows = (uint32_t)Dp * 16;        // bytes between 8-row groups of the tile
  uint8_t* tile = sm + S.tile;
  uint8_t* qs = sm + S.qs;
  uint8_t* pt = sm + S.pt;
  uint8_t* ptm = pt + kTileRows * G * 2;               // (P * row scale)^T for the FP8 dims
  uint64_t* rowf8 = reinterpret_cast<uint64_t*>(sm + S.rowf8);
  uint64_t* rowbf = reinterpret_cast<uint64_t*>(sm + S.rowbf);
  float* rsc = reinterpret_cast<float*>(sm + S.rsc);
  float* m_t = reinterpret_cast<float*>(sm + S.stats);
  float* l_t = m_t + 32;
  float* m_run = l_t + 32;
  float* l_run = m_run + 32;
  float* alpha = l_run + 32;
  float* beta = alpha + 32;
  float* cmul = beta + 32;
  float* den = cmul + 32;
  float* part = den + 32;                                // [4][32]
  float* m_tot = part + 128;                             // whole-query launch, chunks of > 1 tile
  float* l_tot = m_tot + 32;
  int32_t* pgt = reinterpret_cast<int32_t*>(sm + S.pgt);
  uint64_t* bar_qk = reinterpret_cast<uint64_t*>(sm + S.bars);
  uint64_t* bar_pv = bar_qk + 1;
  uint64_t* bar_drain = bar_qk + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_qk + 3);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i = kSplit ? (int)blockIdx.z : (int)blockIdx.x;
  const int h0 = blockIdx.y * G;
  const int c0 = kSplit ? (int)blockIdx.x : 0;         // split launch: this CTA's chunk
  QueryGeom g;
  const bool reporter = tid == 0 && blockIdx.y == 0 && (!kSplit || blockIdx.x == 0);
  // The kernel is launched with programmatic serialization: its CTAs may be
  // resident before the previous grid on the stream (the top-k selection,
  // or the append on an HCA layer) has finished.  Without state_ready every
  // thread waits for that grid here.  With it, the query's length, q, the
  // page table and the window rows are read first; the wait comes before
  // the first top-k list or compressed entry is read (before the first
  // tile's rows are resolved, or, for a tile of window rows only, once that
  // tile has been gathered) and before anything is written.
  const bool early = a.state_ready != 0;
  if (!early) tc::griddep_wait();
  if (!query_geom(a, i, g, reporter)) return;
  if (kSplit) {
    if (g.n_chunks > a.chunks_max) {
      if (reporter) set_err(L, kErrBounds, 4000000 + i);
      return;
    }
    if (c0 >= g.n_chunks) {
      if (a.cluster_fold) {      // no rows: an empty partial, and this CTA's share of the fold
        float2* ml_stage = reinterpret_cast<float2*>(tile + (int64_t)G * D * 4);
        for (int x = tid; x < G; x += kAttThreads) ml_stage[x] = make_float2(-INFINITY, 0.f);
        cluster_fold(G, H, D, a.sink, static_cast<uint16_t*>(a.out), g.n_chunks, i, h0,
                     reinterpret_cast<const float*>(tile), ml_stage, reinterpret_cast<float2*>(pt));
      }
      return;
    }
  }
  const int tt0 = kSplit ? c0 * g.chunk : 0;
  const int tt_end = kSplit ? min(tt0 + g.chunk, g.n_tiles) : g.n_tiles;
  const bool multi = tt_end - tt0 > 1 || !kSplit;       // tiles are folded on chip
  const bool two_level = !kSplit && g.chunk > 1;       // chunk results fold into a total on chip
  const int64_t pages_needed = (g.n_entries + L.rows_per_page(a.layer) - 1) / L.rows_per_page(a.layer);
  const int n_pgt = (int)(pages_needed < kPgtCache ? pages_needed : kPgtCache);

  // TMEM columns: S over the FP8 dims, S over the RoPE dims, the tile's
  // output accumulators (per 128-dim block one for the FP8 dims and, where
  // the block holds RoPE dims, one for those), then (tiles folded on chip)
  // the running output of the chunk, one accumulator per 128-dim block, and
  // (two-level fold) the total.
  const int n_dc = Dp / 128;
  const int dmain = D - R;
  const int dc_r0 = dmain / 128;                        // first chunk holding RoPE dims
  const int n_acc = n_dc + (n_dc - dc_r0);
  const uint32_t col_s = 0, col_sr = G, col_ot = 2 * G, col_orun = 2 * G + n_acc * G;
  const uint32_t col_otot = col_orun + n_dc * G;
  const int cols_needed = (int)col_orun + (multi ? n_dc * G : 0) + (two_level ? n_dc * G : 0);
  uint32_t n_cols = 32;
  while ((int)n_cols < cols_needed) n_cols <<= 1;

  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, n_cols);
    tc::tmem_relinquish();
  }
  if (tid == 32) {
    tc::mbar_init(bar_qk, 1);
    tc::mbar_init(bar_pv, 1);
    tc::mbar_init(bar_drain, 1);
    tc::fence_mbar_init();
  }
  if (tid < 32) { m_run[tid] = -INFINITY; l_run[tid] = 0.f; m_tot[tid] = -INFINITY; l_tot[tid] = 0.f; }

  // gather geometry: chunks of a row are FP8 (16 dims) then BF16 (8 dims);
  // item `it` of a tile = 8 rows x 4 chunks, one 16-byte load per lane
  const int nc8 = dmain / 16, nc = nc8 + R / 8;
  const int n_items = 16 * ((nc + 3) / 4);
  auto gather_load = [&](int it) -> uint4 {
    const int r = 8 * (it & 15) + (lane & 7), c = 4 * (it >> 4) + (lane >> 3);
    if (c < nc8) {
      const uint8_t* p = reinterpret_cast<const uint8_t*>(rowf8[r]);
      if (p != nullptr) return ld_nc16(p + 16 * c);
    } else if (c < nc) {
      const uint16_t* p = reinterpret_cast<const uint16_t*>(rowbf[r]);
      if (p != nullptr) return ld_nc16(p + 8 * (c - nc8));
    }
    return make_uint4(0, 0, 0, 0);
  };
  // dequantise (FP8 -> BF16 is exact) and store in the core-matrix order
  auto gather_store = [&](int it, const uint4& v) {
    const int r = 8 * (it & 15) + (lane & 7), c = 4 * (it >> 4) + (lane >> 3);
    uint8_t* dst = tile + (r >> 3) * sbo_rows + (r & 7) * 16;
    if (c < nc8) {
      const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
      uint32_t pk[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t b2 = (wv[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
        const __half2_raw h2 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)b2, __NV_E4M3);
        const float2 f = __half22float2(__half2(h2));
        pk[e] = (uint32_t)bf16_rn(f.x) | ((uint32_t)bf16_rn(f.y) << 16);
      }
      *reinterpret_cast<uint4*>(dst + (2 * c) * 128) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      *reinterpret_cast<uint4*>(dst + (2 * c + 1) * 128) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    } else if (c < nc) {
      *reinterpret_cast<uint4*>(dst + (dmain / 8 + c - nc8) * 128) = v;
    }
  };

  // The request's page-table entries and the query heads h0 .. h0+G-1 (in
  // the K-major core-matrix order) go to shared memory by cp.async (no
  // registers), issued first; warps 0-3 then resolve the first tile's row
  // addresses while warps
  // 4-7 tabulate cos / sin of the query position and clear the tile's padding
  // dims.  All warps then gather the first tile in one round of loads, and
  // the query's RoPE dims are rotated in place once its copies have landed.
  {
    // the request's page-table entries that hold its completed entries, one
    // cp.async group (waited for before the rows are resolved)
    const int32_t* ptg = L.page_table(g.req);
    for (int x = tid; x < n_pgt; x += kAttThreads)
      asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(tc::smem_u32(pgt + x)), "l"(ptg + x) : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  {
    const uint16_t* qg = static_cast<const uint16_t*>(a.q) + ((int64_t)i * H + h0) * D;
    for (int x = tid; x < G * (Dp / 8); x += kAttThreads) {
      const int hh = x / (Dp / 8), c = x % (Dp / 8);
      uint8_t* dst = qs + (hh >> 3) * sbo_rows + c * 128 + (hh & 7) * 16;
      if (h0 + hh < H && 8 * c < D)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(dst)), "l"(qg + (int64_t)hh * D + 8 * c)
                     : "memory");
      else
        *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  asm volatile("cp.async.wait_group 1;" ::: "memory");  // its page-table group has landed (the query's may not)
  __syncthreads();
  const bool list_rows = (int64_t)tt0 * kTileRows < g.n_list;   // the first tile holds top-k / entry rows
  if (early && list_rows) tc::griddep_wait();
  float2* cs = reinterpret_cast<float2*>(pt);         // P^T is first written by the first tile's softmax
  const float* scp = nullptr;         // warps 0-3: FP8 scale of row tid of the tile being fetched
  float scv = 0.f;                    // its value, loaded with the tile's gather
  int any = 0;
  if (warp < 4) {
    any = resolve_row(a, g, i, tt0, tid, rowf8, rowbf, &scp, pgt, n_pgt) ? 1 : 0;
  } else {
    const int qt = tid - 128;
    for (int p = qt; p < R / 2; p += 128) {
      float c = 1.f, sn = 0.f;
      rope_pair(c, sn, L.theta()[p], g.t);       // rotating (1, 0) gives (cos, sin)
      cs[p] = make_float2(c, sn);
    }
    // padding dims [D, Dp) of the tile stay zero
    const int npad = (Dp - D) / 8;
    for (int x = qt; x < kTileRows * npad; x += 128) {
      const int r = x % kTileRows, c = D / 8 + x / kTileRows;
      *reinterpret_cast<uint4*>(tile + (r >> 3) * sbo_rows + c * 128 + (r & 7) * 16) = make_uint4(0, 0, 0, 0);
    }
  }
  bool tile_valid = __syncthreads_count(any) > 0;
  {   // the first tile: every warp, all its loads in flight at once
    uint4 buf[kMaxLoads];
#pragma unroll
    for (int u = 0; u < kMaxLoads; ++u) {
      const int it = warp + 8 * u;
      buf[u] = it < n_items ? gather_load(it) : make_uint4(0, 0, 0, 0);
    }
    scv = scp != nullptr ? __ldg(scp) : 0.f;
#pragma unroll
    for (int u = 0; u < kMaxLoads; ++u) {
      const int it = warp + 8 * u;
      if (it < n_items) gather_store(it, buf[u]);
    }
    if (warp < 4) rsc[tid] = scv;
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();                                      // every thread's query copies have landed
  for (int x = tid; x < G * (R / 2); x += kAttThreads) {
    // RoPE dims of the query: rotate the BF16 input at t, round to BF16
    const int hh = x / (R / 2), p = x % (R / 2);
    const int d = dmain + 2 * p;
    uint32_t* wp = reinterpret_cast<uint32_t*>(qs + (hh >> 3) * sbo_rows + (d >> 3) * 128 + (hh & 7) * 16 + (d & 7) * 2);
    const uint32_t v = *wp;
    const float2 w = cs[p];
    const float x0 = bf16_val((uint16_t)(v & 0xFFFFu)), x1 = bf16_val((uint16_t)(v >> 16));
    *wp = (uint32_t)bf16_rn(x0 * w.x - x1 * w.y) | ((uint32_t)bf16_rn(x0 * w.y + x1 * w.x) << 16);
  }
  if (early && !list_rows) tc::griddep_wait();          // a window-only tile: gathered, nothing written yet
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  const bool tw = warp < 4 * (G / 16);                  // this warp reads TMEM: lanes (warp%4)*32.., heads hb..hb+15
  const int hb = 16 * (warp >> 2);
  const uint32_t id_qk = tc::idesc_bf16(128, G, false, false);
  const uint32_t id_pv = tc::idesc_bf16(128, G, true, true);
  bool ok = true;
  int n_done = 0;                                        // tiles whose PV has been issued
  bool pend_fold = false;                                // the last tile's (m_t, l_t, O_t) await their fold
  bool chunk_has = false;                                // the current chunk holds a tile with rows

  // Fold the pending tile into the chunk's running (m, l, O) (its PV has
  // completed).  All threads.
  auto fold_pending = [&]() {
    if (tid < G) {
      float mn, al, be;
      fold_coef(m_run[tid], m_t[tid], mn, al, be);
      alpha[tid] = al;
      beta[tid] = be;
      m_run[tid] = mn;
      l_run[tid] = fold_val(l_run[tid], al, l_t[tid], be);
    }
    __syncthreads();
    if (tw) {
      for (int dc = 0; dc < n_dc; ++dc) {
        const int d = dc * 128 + (warp & 3) * 32 + lane;
        const bool has_rope = dc >= dc_r0;
        uint32_t om[16], orp[16], orun[16];
        tc::tmem_ld_x16(tmem + lane_base + col_ot + dc * G + hb, om);
        if (has_rope) tc::tmem_ld_x16(tmem + lane_base + col_ot + (n_dc + dc - dc_r0) * G + hb, orp);
        tc::tmem_ld_x16(tmem + lane_base + col_orun + dc * G + hb, orun);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float ot = __uint_as_float(d < dmain ? om[e] : orp[e]);
          orun[e] = __float_as_uint(fold_val(__uint_as_float(orun[e]), alpha[hb + e], ot, beta[hb + e]));
        }
        tc::tmem_st_x16(tmem + lane_base + col_orun + dc * G + hb, orun);
      }
      tc::tmem_wait_st();
    }
    pend_fold = false;
  };
  // Two-level fold: the finished chunk's (m, l, O) into the total (an empty
  // chunk is skipped, as the fold kernel skips its partial); the chunk
  // result starts again empty.  All threads.
  auto fold_chunk = [&]() {
    __syncthreads();                                     // alpha / beta of the last tile fold are read
    if (chunk_has) {
      if (tid < G) {
        float mn, al, be;
        fold_coef(m_tot[tid], m_run[tid], mn, al, be);
        alpha[tid] = al;
        beta[tid] = be;
        m_tot[tid] = mn;
        l_tot[tid] = fold_val(l_tot[tid], al, l_run[tid], be);
      }
      __syncthreads();
      if (tw) {
        for (int dc = 0; dc < n_dc; ++dc) {
          uint32_t orun[16], otot[16];
          tc::tmem_ld_x16(tmem + lane_base + col_orun + dc * G + hb, orun);
          tc::tmem_ld_x16(tmem + lane_base + col_otot + dc * G + hb, otot);
          tc::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e)
            otot[e] = __float_as_uint(fold_val(__uint_as_float(otot[e]), alpha[hb + e], __uint_as_float(orun[e]),
                                               beta[hb + e]));
          tc::tmem_st_x16(tmem + lane_base + col_otot + dc * G + hb, otot);
        }
        tc::tmem_wait_st();
      }
      __syncthreads();
    }
    if (tid < G) { m_run[tid] = -INFINITY; l_run[tid] = 0.f; }
    chunk_has = false;
    __syncthreads();
  };

  // The next tile's rows are resolved and their loads issued (into buf) as
  // soon as the current tile's PV is issued, so that they fly during the row
  // sums, the PV and the fold; buf_tile is the tile whose loads buf holds.
  uint4 buf[kMaxLoads];
  int buf_tile = tt0;                                    // the first tile was gathered in the prologue
  bool next_resolved = false;
  for (int tt = tt0; tt < tt_end && ok; ++tt) {
    if (two_level && tt > tt0 && tt % g.chunk == 0) {
      // a chunk ends before tile tt: its last tile and then the chunk fold in
      if (pend_fold) {
        if (n_done > 0) ok = tc::mbar_wait(bar_pv, (n_done - 1) & 1);
        ok = __syncthreads_and(ok) != 0;
        if (!ok) break;
        tc::tc_fence_after();
        fold_pending();
      }
      fold_chunk();
    }
    if (tile_valid) {
      // the previous PV has finished: tile buffer, P^T and O_t are free
      if (n_done > 0) ok = tc::mbar_wait(bar_pv, (n_done - 1) & 1);
      ok = __syncthreads_and(ok) != 0;
      if (!ok) break;
      tc::tc_fence_after();
      // -- gather: the loads were issued with the previous tile, unless it
      //    had no rows (the first tile was gathered in the prologue)
      const bool fetch = tt != tt0;
      if (fetch && buf_tile != tt) {
#pragma unroll
        for (int u = 0; u < kMaxLoads; ++u) {
          const int it = warp + 8 * u;
          buf[u] = it < n_items ? gather_load(it) : make_uint4(0, 0, 0, 0);
        }
        scv = scp != nullptr ? __ldg(scp) : 0.f;
        buf_tile = tt;
      }
      // -- fold the previous tile while the loads fly
      if (pend_fold) fold_pending();
      // -- dequantise and store the tile
      if (fetch) {
#pragma unroll
        for (int u = 0; u < kMaxLoads; ++u) {
          const int it = warp + 8 * u;
          if (it < n_items) gather_store(it, buf[u]);
        }
        if (warp < 4) rsc[tid] = scv;
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      __syncthreads();
      tc::tc_fence_after();
      // -- QK: S^T[rows x heads]
      if (warp == 0) {
        if (tc::elect_one()) {
          const uint32_t ta = tc::smem_u32(tile), tq = tc::smem_u32(qs);
          for (int ks = 0; ks < Dp / 16; ++ks) {
            const bool main = 16 * ks < dmain;                // dmain is a multiple of 16
            const int k0 = main ? 0 : dmain / 16;
            tc::mma_bf16(tmem + (main ? col_s : col_sr), tc::smem_desc(ta + ks * 256, 128, sbo_rows),
                         tc::smem_desc(tq + ks * 256, 128, sbo_rows), id_qk, ks > k0 ? 1u : 0u);
          }
          tc::mma_commit(bar_qk);
        }
        __syncwarp();
      }
      // -- logits u = scale * (row scale * S_fp8 + S_rope); empty rows -inf
      const int r = (warp & 3) * 32 + lane;
      float u[16];
      if (tw) {
        ok = tc::mbar_wait(bar_qk, n_done & 1);
        tc::tc_fence_after();
        uint32_t sv[16], sr[16];
        tc::tmem_ld_x16(tmem + lane_base + col_s + hb, sv);
        tc::tmem_ld_x16(tmem + lane_base + col_sr + hb, sr);
        tc::tmem_wait_ld();
        const bool valid = rowf8[r] != 0;
        const float rs = rsc[r];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          u[e] = valid ? fmaf(rs, __uint_as_float(sv[e]), __uint_as_float(sr[e])) * a.scale : -INFINITY;
        // max over this warp's 32 rows, per head; then over the 4 row warps
        const float mx = warp_reduce16<true>(u, lane);
        if ((lane & 1) == 0) part[(warp & 3) * 32 + hb + (lane >> 1)] = mx;
      }
      ok = __syncthreads_and(ok) != 0;
      if (!ok) break;
      if (tid < G) m_t[tid] = fmaxf(fmaxf(part[tid], part[32 + tid]), fmaxf(part[64 + tid], part[96 + tid]));
      __syncthreads();
      // -- p = exp(u - m_t): P^T and (P * row scale)^T in BF16 for PV, fp32 p for the sums
      float pv[16];
      if (tw) {
        const float rs = rsc[r];
#pragma unroll
        for (int hg = 0; hg < 2; ++hg) {
          uint32_t pk[4], pm[4];
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const int h = hb + hg * 8 + e;
            const float p0 = expf(u[hg * 8 + e] - m_t[h]);
            const float p1 = expf(u[hg * 8 + e + 1] - m_t[h + 1]);
            pv[hg * 8 + e] = p0;
            pv[hg * 8 + e + 1] = p1;
            pk[e >> 1] = (uint32_t)bf16_rn(p0) | ((uint32_t)bf16_rn(p1) << 16);
            pm[e >> 1] = (uint32_t)bf16_rn(p0 * rs) | ((uint32_t)bf16_rn(p1 * rs) << 16);
          }
          const int hgl = (hb >> 3) + hg;
          *reinterpret_cast<uint4*>(pt + hgl * 2048 + (r >> 3) * 128 + (r & 7) * 16) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(ptm + hgl * 2048 + (r >> 3) * 128 + (r & 7) * 16) =
              make_uint4(pm[0], pm[1], pm[2], pm[3]);
        }
      }
      tc::fence_proxy_async_smem();
      tc::tc_fence_before();
      __syncthreads();
      tc::tc_fence_after();
      // -- PV: O_t^T[dims x heads] = V^T P^T
      if (warp == 0) {
        if (tc::elect_one()) {
          const uint32_t ta = tc::smem_u32(tile), tp = tc::smem_u32(pt), tpm = tc::smem_u32(ptm);
          for (int x = 0; x < n_acc; ++x) {
            const bool main = x < n_dc;
            const int dc = main ? x : dc_r0 + (x - n_dc);
            for (int ks = 0; ks < kTileRows / 16; ++ks)
              tc::mma_bf16(tmem + col_ot + x * G,
                           tc::smem_desc(ta + dc * 16 * 128 + ks * 2 * sbo_rows, sbo_rows, 128),
                           tc::smem_desc((main ? tpm : tp) + ks * 256, 128, 2048), id_pv, ks > 0 ? 1u : 0u);
          }
          tc::mma_commit(bar_pv);
        }
        __syncwarp();
      }
      ++n_done;
      // -- the next tile: rows resolved (the current tile no longer reads
      //    them) and loads issued now
      if (tt + 1 < tt_end) {
        int nany = 0;
        if (warp < 4) nany = resolve_row(a, g, i, tt + 1, tid, rowf8, rowbf, &scp, pgt, n_pgt) ? 1 : 0;
        tile_valid = __syncthreads_count(nany) > 0;
        next_resolved = true;
        if (tile_valid) {
#pragma unroll
          for (int u = 0; u < kMaxLoads; ++u) {
            const int it = warp + 8 * u;
            buf[u] = it < n_items ? gather_load(it) : make_uint4(0, 0, 0, 0);
          }
          scv = scp != nullptr ? __ldg(scp) : 0.f;
          buf_tile = tt + 1;
        }
      }
      // -- l_t: row sums of p per head, in a fixed order (warp tree, then the 4 row warps)
      if (tw) {
        const float sm_ = warp_reduce16<false>(pv, lane);
        if ((lane & 1) == 0) part[(warp & 3) * 32 + hb + (lane >> 1)] = sm_;
      }
      __syncthreads();
      if (tid < G) l_t[tid] = ((part[tid] + part[32 + tid]) + part[64 + tid]) + part[96 + tid];
      pend_fold = true;
      chunk_has = true;
    }
    // -- addresses of the next tile's rows (after a tile without rows)
    if (tt + 1 < tt_end && !next_resolved) {
      int nany = 0;
      if (warp < 4) nany = resolve_row(a, g, i, tt + 1, tid, rowf8, rowbf, &scp, pgt, n_pgt) ? 1 : 0;
      tile_valid = __syncthreads_count(nany) > 0;
    }
    next_resolved = false;
  }

  if (ok && n_done > 0) ok = tc::mbar_wait(bar_pv, (n_done - 1) & 1);
  ok = __syncthreads_and(ok) != 0;
  // split launch: where this chunk's partial goes -- the workspace, or (the
  // cluster fold) this CTA's shared memory, the tile buffer being free now
  // that the last PV has completed: O_c [G][D] then (m_c, l_c) [G]
  const bool cfold = kSplit && a.cluster_fold != 0;
  float* const o_stage = reinterpret_cast<float*>(tile);
  float2* const ml_stage = reinterpret_cast<float2*>(tile + (int64_t)G * D * 4);
  float* const wo = !kSplit ? nullptr
                    : cfold ? o_stage : a.ws_o + (((int64_t)i * a.chunks_max + c0) * H + h0) * D;    // [head - h0][D]
  float2* const wml = !kSplit ? nullptr
                      : cfold ? ml_stage : a.ws_ml + ((int64_t)i * a.chunks_max + c0) * H + h0;     // [head - h0]
  if (ok && kSplit && n_done == 0) {
    // ---- split launch, a chunk without rows: an empty partial
    if (tid < G && h0 + tid < H) wml[tid] = make_float2(-INFINITY, 0.f);
  } else if (ok && kSplit && multi) {
    // ---- split launch, a chunk of several tiles: fold its last tile, then
    // the chunk's (m, l, O)
    tc::tc_fence_after();
    if (pend_fold) fold_pending();
    if (tid < G && h0 + tid < H) wml[tid] = make_float2(m_run[tid], l_run[tid]);
    if (tw) {
      for (int dc = 0; dc < n_dc; ++dc) {
        uint32_t orun[16];
        tc::tmem_ld_x16(tmem + lane_base + col_orun + dc * G + hb, orun);
        tc::tmem_wait_ld();
        const int d = dc * 128 + (warp & 3) * 32 + lane;
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int h = h0 + hb + e;
          if (h < H && d < D) wo[(int64_t)(hb + e) * D + d] = __uint_as_float(orun[e]);
        }
      }
    }
  } else if (ok && kSplit) {
    // ---- split launch, a chunk of one tile: the tile's partial is the
    // chunk's (folding into an empty result is exact)
    tc::tc_fence_after();
    if (tid < G && h0 + tid < H) wml[tid] = make_float2(m_t[tid], l_t[tid]);
    if (tw) {
      // two 128-dim blocks per TMEM wait
      for (int dc0 = 0; dc0 < n_dc; dc0 += 2) {
        uint32_t om[2][16], orp[2][16];
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          const int dc = dc0 + q2;
          if (dc < n_dc) {
            tc::tmem_ld_x16(tmem + lane_base + col_ot + dc * G + hb, om[q2]);
            if (dc >= dc_r0) tc::tmem_ld_x16(tmem + lane_base + col_ot + (n_dc + dc - dc_r0) * G + hb, orp[q2]);
          }
        }
        tc::tmem_wait_ld();
#pragma unroll
        for (int q2 = 0; q2 < 2; ++q2) {
          const int dc = dc0 + q2;
          if (dc >= n_dc) break;
          const int d = dc * 128 + (warp & 3) * 32 + lane;
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const int h = h0 + hb + e;
            if (h < H && d < D) wo[(int64_t)(hb + e) * D + d] = __uint_as_float(d < dmain ? om[q2][e] : orp[q2][e]);
          }
        }
      }
    }
  } else if (ok && two_level) {
    // ---- whole-query launch, two-level fold: the last tile, the last chunk,
    // then out = O e^{m-mu} / (l e^{m-mu} + e^{sink-mu}) from the total
    tc::tc_fence_after();
    if (pend_fold) fold_pending();
    fold_chunk();
    if (tid < G) {
      const int h = h0 + tid;
      float cm, dn;
      finish_coef(m_tot[tid], h < H ? a.sink[h] : 0.f, l_tot[tid], cm, dn);
      cmul[tid] = cm;
      den[tid] = dn;
    }
    __syncthreads();
    if (tw) {
      for (int dc = 0; dc < n_dc; ++dc) {
        const int d = dc * 128 + (warp & 3) * 32 + lane;
        uint32_t otot[16];
        tc::tmem_ld_x16(tmem + lane_base + col_otot + dc * G + hb, otot);
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int h = h0 + hb + e;
          if (h < H && d < D)
            static_cast<uint16_t*>(a.out)[((int64_t)i * H + h) * D + d] =
                finish_val(__uint_as_float(otot[e]), cmul[hb + e], den[hb + e]);
        }
      }
    }
  } else if (ok && !kSplit) {
    // ---- whole-query launch: fold the last tile, then out = O e^{m-mu} / (l e^{m-mu} + e^{sink-mu})
    tc::tc_fence_after();
    if (tid < G) {
      float mr = m_run[tid], lr = l_run[tid];
      if (pend_fold) {
        float mn, al, be;
        fold_coef(mr, m_t[tid], mn, al, be);
        alpha[tid] = al;
        beta[tid] = be;
        lr = fold_val(lr, al, l_t[tid], be);
        mr = mn;
      }
      const int h = h0 + tid;
      float cm, dn;
      finish_coef(mr, h < H ? a.sink[h] : 0.f, lr, cm, dn);
      cmul[tid] = cm;
      den[tid] = dn;
    }
    __syncthreads();
    if (tw) {
      for (int dc = 0; dc < n_dc; ++dc) {
        const int d = dc * 128 + (warp & 3) * 32 + lane;
        const bool has_rope = dc >= dc_r0;
        uint32_t om[16], orp[16], orun[16];
        tc::tmem_ld_x16(tmem + lane_base + col_orun + dc * G + hb, orun);
        if (pend_fold) {
          tc::tmem_ld_x16(tmem + lane_base + col_ot + dc * G + hb, om);
          if (has_rope) tc::tmem_ld_x16(tmem + lane_base + col_ot + (n_dc + dc - dc_r0) * G + hb, orp);
        }
        tc::tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int h = h0 + hb + e;
          float o = __uint_as_float(orun[e]);
          if (pend_fold) o = fold_val(o, alpha[hb + e], __uint_as_float(d < dmain ? om[e] : orp[e]), beta[hb + e]);
          if (h < H && d < D)
            static_cast<uint16_t*>(a.out)[((int64_t)i * H + h) * D + d] = finish_val(o, cmul[hb + e], den[hb + e]);
        }
      }
    }
  } else if (!ok) {
    if (tid == 0) set_err(L, kErrTimeout, 3000000 + i);
    if (cfold && tid < G) ml_stage[tid] = make_float2(-INFINITY, 0.f);   // the fold still runs; the error stands
  }
  tc::griddep_launch_dependents();                      // the fold (or the next step) may start launching
  if (warp == 0) {   // no tcgen05 operation of this CTA is in flight when TMEM is released
    if (tc::elect_one()) tc::mma_commit(bar_drain);
    __syncwarp();
    tc::mbar_wait(bar_drain, 0, 200000000ull);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, n_cols);
  if (cfold)
    cluster_fold(G, H, D, a.sink, static_cast<uint16_t*>(a.out), g.n_chunks, i, h0, o_stage, ml_stage,
                 reinterpret_cast<float2*>(pt));
}

// Split launch, second step: fold the chunk partials of (query blockIdx.y,
// head blockIdx.x) in chunk order; thread x owns dims 4x .. 4x+3.
__global__ void __launch_bounds__(128) attn_fold_kernel(AttnArgs a) {
  const Layout& L = a.L;
  const int h = blockIdx.x, i = blockIdx.y, H = L.H, D = L.D;
  const int d4 = threadIdx.x;
  // The request id and its length are final before the partial kernel
  // (the previous grid) starts, so the query's geometry is read while that
  // grid finishes; the partials only after the wait.
  QueryGeom g;
  const bool have = 4 * d4 < D && query_geom(a, i, g, false);   // a bad query is recorded by the partial kernel
  tc::griddep_wait();                                   // the partials are complete from here on
  if (!have || g.n_chunks > a.chunks_max) return;
  float m = -INFINITY, l = 0.f;
  float o[4] = {0.f, 0.f, 0.f, 0.f};
  const int64_t base = (int64_t)i * a.chunks_max;
  for (int t0 = 0; t0 < g.n_chunks; t0 += kFoldBatch) {
    float2 ml[kFoldBatch];
    float4 v[kFoldBatch];
#pragma unroll
    for (int x = 0; x < kFoldBatch; ++x) {
      if (t0 + x < g.n_chunks) {
        ml[x] = a.ws_ml[(base + t0 + x) * H + h];
        v[x] = reinterpret_cast<const float4*>(a.ws_o + ((base + t0 + x) * H + h) * D)[d4];
      } else {
        ml[x] = make_float2(-INFINITY, 0.f);
        v[x] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
#pragma unroll
    for (int x = 0; x < kFoldBatch; ++x) {
      if (ml[x].x == -INFINITY) continue;
      float mn, al, be;
      fold_coef(m, ml[x].x, mn, al, be);
      l = fold_val(l, al, ml[x].y, be);
      o[0] = fold_val(o[0], al, v[x].x, be);
      o[1] = fold_val(o[1], al, v[x].y, be);
      o[2] = fold_val(o[2], al, v[x].z, be);
      o[3] = fold_val(o[3], al, v[x].w, be);
      m = mn;
    }
  }
  float cm, dn;
  finish_coef(m, a.sink[h], l, cm, dn);
  if (a.f32) {
    *reinterpret_cast<float4*>(static_cast<float*>(a.out) + ((int64_t)i * H + h) * D + 4 * d4) =
        make_float4(finish_f32(o[0], cm, dn), finish_f32(o[1], cm, dn), finish_f32(o[2], cm, dn),
                    finish_f32(o[3], cm, dn));
    return;
  }
  uint2 pk;
  pk.x = (uint32_t)finish_val(o[0], cm, dn) | ((uint32_t)finish_val(o[1], cm, dn) << 16);
  pk.y = (uint32_t)finish_val(o[2], cm, dn) | ((uint32_t)finish_val(o[3], cm, dn) << 16);
  *reinterpret_cast<uint2*>(static_cast<uint16_t*>(a.out) + ((int64_t)i * H + h) * D + 4 * d4) = pk;
}

cudaError_t launch_attn_fold(const AttnArgs& a, cudaStream_t st) {
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(a.L.H, a.n);
  cfg.blockDim = dim3((a.L.D / 4 + 31) / 32 * 32);
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, attn_fold_kernel, a);
  note_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

size_t attn_tc_smem_bytes(int D, int G) { return (size_t)attn_smem(D, G).total + 1024; }

// Dynamic shared memory of an attention launch, and a carveout no larger
// than it needs: what the carveout leaves is the SM's L1, which holds the
// row gathers in flight.
template <bool kSplit>
static cudaError_t attn_smem_attrs(size_t smem) {
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel<kSplit>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int pct = (int)(((smem + 1024) * 100 + 228 * 1024 - 1) / (228 * 1024));
  return cudaFuncSetAttribute(attn_tc_kernel<kSplit>, cudaFuncAttributePreferredSharedMemoryCarveout,
                              pct < 100 ? pct : 100);
}

int attn_tiles_max(const Layout& L, int layer, int k) {
  const int64_t rows = (layer < L.n_csa ? (int64_t)k : (int64_t)L.max_pages_per_req * kHcaPerPage) + kWindow;
  return (int)((rows + kTileRows - 1) / kTileRows);
}

int attn_chunks_max(const Layout& L, int layer, int k) {
  const int t = attn_tiles_max(L, layer, k);
  if (layer < L.n_csa) return t;
  int m = 0;                     // the most chunks any query of at most t tiles has
  for (int n = 1; n <= t; ++n) {
    const int c = attn_chunk_tiles(false, n);
    m = (n + c - 1) / c > m ? (n + c - 1) / c : m;
  }
  return m;
}

size_t attn_workspace_bytes(const Layout& L, int layer, int n, int k) {
  const int64_t units = (int64_t)n * attn_chunks_max(L, layer, k) * L.H;
  return (size_t)(units * L.D * 4 + units * 8);
}

// How many clusters of C split-launch CTAs (smem bytes each) the device can
// hold at once; asked once per (device, C, smem) and remembered.
static cudaError_t cluster_fold_capacity(int C, size_t smem, int* out) {
  static std::mutex mu;
  struct Entry { int dev, C; size_t smem; int n; };
  static std::vector<Entry> seen;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& x : seen)
    if (x.dev == dev && x.C == C && x.smem == smem) { *out = x.n; return cudaSuccess; }
  if (C > 8) {
    e = cudaFuncSetAttribute(attn_tc_kernel<true>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  e = attn_smem_attrs<true>(smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = (unsigned)C;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)C, 1, 1);
  cfg.blockDim = dim3(kAttThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  e = cudaOccupancyMaxActiveClusters(&n, attn_tc_kernel<true>, &cfg);
  if (e != cudaSuccess) {       // not available: the workspace path
    (void)cudaGetLastError();
    n = 0;
  }
  seen.push_back(Entry{dev, C, smem, n});
  *out = n;
  return cudaSuccess;
}

cudaError_t launch_attn_tc(const Layout& L, int layer, int n, const int32_t* req_ids, const uint16_t* q,
                           const int32_t* topk, int k, const float* sink, float scale, uint16_t* out, int G,
                           void* ws, cudaStream_t st, bool state_ready, int q_per_req, const char* win_snap) {
  const size_t sm = attn_tc_smem_bytes(L.D, G);
  if (sm > 227 * 1024) return cudaErrorInvalidValue;
  const bool split = ws != nullptr;
  AttnArgs a{L, layer, n, req_ids, q, topk, k, sink, scale, out, G, nullptr, nullptr, 0, 0, state_ready ? 1 : 0,
             q_per_req, win_snap};
  const int n_hg = (L.H + G - 1) / G;
  // programmatic dependent launch: the kernel may start before the previous
  // grid on the stream ends and waits for it (griddepcontrol) where it must
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kAttThreads);
  cfg.dynamicSmemBytes = sm;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  if (!split) {
    cudaError_t e = attn_smem_attrs<false>(sm);
    if (e != cudaSuccess) return e;
    cfg.gridDim = dim3(n, n_hg);
    e = cudaLaunchKernelEx(&cfg, attn_tc_kernel<false>, a);
    note_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  a.chunks_max = attn_chunks_max(L, layer, k);
  a.ws_o = static_cast<float*>(ws);
  a.ws_ml = reinterpret_cast<float2*>(static_cast<char*>(ws) + (int64_t)n * a.chunks_max * L.H * L.D * 4);
  cudaError_t e = attn_smem_attrs<true>(sm);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3(a.chunks_max, n_hg, n);
  // The fold in the cluster when every cluster of the launch (one per query
  // and head group, a CTA per chunk) can be resident at once; otherwise the
  // partials go through the workspace to attn_fold_kernel.  Both give the
  // same bits.
  int resident = 0;
  if (a.chunks_max >= 2 && a.chunks_max <= kClusterFoldMax && (L.D % 4) == 0) {
    e = cluster_fold_capacity(a.chunks_max, sm, &resident);
    if (e != cudaSuccess) return e;
  }
  if (resident >= n_hg * n) {
    cudaLaunchAttribute at2[2];
    at2[0] = at[0];
    at2[1].id = cudaLaunchAttributeClusterDimension;
    at2[1].val.clusterDim.x = (unsigned)a.chunks_max;
    at2[1].val.clusterDim.y = 1;
    at2[1].val.clusterDim.z = 1;
    cfg.attrs = at2;
    cfg.numAttrs = 2;
    a.cluster_fold = 1;
    e = cudaLaunchKernelEx(&cfg, attn_tc_kernel<true>, a);
    note_launch();
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
  }
  e = cudaLaunchKernelEx(&cfg, attn_tc_kernel<true>, a);
  note_launch();
  if (e != cudaSuccess) return e;
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attn_fold(a, st);
}

// ---- scratch for csa_hca_decode_attn_noalloc
//
// For callers that must not allocate device memory: the split launch's
// partials go to this file-scope array instead of a caller workspace.  Every
// GPU that loads the library holds it until the process exits.  All calls
// share it: the partial kernel writes every (tile, head) slot the fold kernel
// reads, so nothing needs clearing between calls, but calls whose kernels
// overlap on the GPU race on it.
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;
constexpr int kNoAllocMaxDevices = 64;
static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

size_t attn_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Device address of g_noalloc_scratch on the current device.  In host code
// the array's name is only a host-side stand-in, so the address is looked up
// with cudaGetSymbolAddress, once per device (by the first call on it), with
// that device current.
cudaError_t attn_noalloc_scratch(void** out) {
  static std::mutex mu;
  static void* addr[kNoAllocMaxDevices] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess) return e;
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace csa
