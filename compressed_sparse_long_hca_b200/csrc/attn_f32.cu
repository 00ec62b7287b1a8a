// Multi-query decode attention for caches in the fp32 storage format
// (csa_hca_decode_attn on a CSA_FMT_F32 cache), on the CUDA cores.
//
// Page "V4终于终于终于终于是来了", sections "CSA——压缩稀疏注意力" and
// "HCA——重度压缩注意力": the same attention as the tensor-core kernel -- the
// query's selected (CSA) or all (HCA) compressed entries, then the window's
// raw tokens, K = V = the stored row, RoPE on the last R dims of q, a sink
// logit per head in the denominator -- with every stored vector, the query
// and the output in fp32.  The tensor cores have no fp32 contraction (tf32
// keeps 10 mantissa bits), so the two products run as fp32 FMA chains here.
//
// Reduction order, as in every format: tiles of 128 rows give
// (m_t, l_t, O_t), folded in order into chunk results, which are folded in
// order, with the shared fold arithmetic, the sink last.  Inside a tile every sum runs in a fixed order:
//   u[h][r]  = scale * (sum over d ascending of q[h][d] k[r][d])
//   l_t[h]   = sum over r ascending of e^{u - m_t}
//   O_t[h][d] = sum over r ascending of e^{u - m_t} v[r][d]
// so that a head's result depends on nothing but the query.  Launch variants:
//   * whole-query launch: one CTA per (query, head group) walks the tiles,
//     folds each into the chunk's running result in shared memory and each
//     chunk result into a total;
//   * split launch: one CTA per (query, head group, chunk) folds the chunk's
//     tiles and writes the chunk result to the workspace, and the shared fold
//     kernel folds them.
// Both give identical bits.
#include "attn_common.cuh"
#include "common.cuh"

namespace csa {

namespace {

constexpr int kF32Threads = 256;
constexpr int kF32Heads = 8;        // heads per CTA

constexpr int kF32MaxOut = kF32Heads * 512 / kF32Threads;   // outputs (head, dim) per thread, D <= 512

// Rows of a tile staged in shared memory at a time (the buffer holds about
// 33 KB); row stride D + 4 floats, so that rows start on different banks.
__host__ __device__ inline int f32_chunk_rows(int D) {
  return D <= 64 ? 128 : D <= 128 ? 64 : D <= 256 ? 32 : 16;
}

struct F32Smem {
  int64_t q, u, rows, run, tot, kv, stats, total;
};

__host__ __device__ inline F32Smem f32_smem(int D) {
  F32Smem s{};
  int64_t o = 0;
  s.q = o;     o += (int64_t)kF32Heads * (D + 4) * 4;      // rotated query heads, stride D + 4
  s.u = o;     o += (int64_t)kF32Heads * kTileRows * 4;    // logits, then e^{u - m_t}
  s.rows = o;  o += (int64_t)kTileRows * 8;                // row addresses (null = no row)
  s.run = o;   o += (int64_t)kF32Heads * D * 4;            // the chunk's running O
  s.tot = o;   o += (int64_t)kF32Heads * D * 4;            // the total O (whole-query launch, chunks > 1 tile)
  s.kv = o;    o += (int64_t)f32_chunk_rows(D) * (D + 4) * 4;   // staged rows
  s.stats = o; o += (int64_t)8 * kF32Heads * 4;            // m_t, l_t, m, l, alpha, beta, m_tot, l_tot
  s.total = o;
  return s;
}

// Address of row `r` of tile `tt` of query i (fp32 storage), null when the
// row does not exist (a -1 in the list, or past the window).
__device__ __forceinline__ const float* f32_row(const AttnArgs& a, const QueryGeom& g, int i, int tt, int r) {
  const Layout& L = a.L;
  const int64_t rr = (int64_t)tt * kTileRows + r;
  if (rr < g.n_list) {
    int64_t j = g.csa ? (int64_t)a.topk[(int64_t)i * a.k + rr] : rr;
    if (j >= g.n_entries) {
      set_err(L, kErrBounds, 2000000 + i);
      return nullptr;
    }
    return j >= 0 ? L.entry_row_f32(g.req, a.layer, j) : nullptr;
  }
  if (rr < g.total) {
    const int64_t p = g.w0 + (rr - g.n_list);
    return reinterpret_cast<const float*>(ring_base(a, g, p)) + (p % kWindow) * L.D;
  }
  return nullptr;
}

}  // namespace

// kSplit: grid (tiles_max, head groups, n); otherwise grid (n, head groups).
template <bool kSplit>
__global__ void __launch_bounds__(kF32Threads) attn_f32_kernel(AttnArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  const Layout& L = a.L;
  const int D = L.D, R = L.R, H = L.H;
  const F32Smem S = f32_smem(D);
  float* qs = reinterpret_cast<float*>(smem_raw + S.q);
  float* us = reinterpret_cast<float*>(smem_raw + S.u);
  const float** rows = reinterpret_cast<const float**>(smem_raw + S.rows);
  float* run = reinterpret_cast<float*>(smem_raw + S.run);
  float* tot = reinterpret_cast<float*>(smem_raw + S.tot);
  float* kv = reinterpret_cast<float*>(smem_raw + S.kv);
  float* m_t = reinterpret_cast<float*>(smem_raw + S.stats);
  float* l_t = m_t + kF32Heads;
  float* m_r = l_t + kF32Heads;
  float* l_r = m_r + kF32Heads;
  float* alpha = l_r + kF32Heads;
  float* beta = alpha + kF32Heads;
  float* m_tot = beta + kF32Heads;
  float* l_tot = m_tot + kF32Heads;
  const int tid = threadIdx.x;
  const int i = kSplit ? (int)blockIdx.z : (int)blockIdx.x;
  const int h0 = blockIdx.y * kF32Heads;
  const int c0 = kSplit ? (int)blockIdx.x : 0;         // split launch: this CTA's chunk
  QueryGeom g;
  const bool reporter = tid == 0 && blockIdx.y == 0 && (!kSplit || blockIdx.x == 0);
  if (!query_geom(a, i, g, reporter)) return;
  if (kSplit) {
    if (g.n_chunks > a.chunks_max) {
      if (reporter) set_err(L, kErrBounds, 4000000 + i);
      return;
    }
    if (c0 >= g.n_chunks) return;
  }
  const int tt0 = kSplit ? c0 * g.chunk : 0;
  const int tt_end = kSplit ? min(tt0 + g.chunk, g.n_tiles) : g.n_tiles;
  const bool two_level = !kSplit && g.chunk > 1;
  const float* q = static_cast<const float*>(a.q) + ((int64_t)i * H) * D;

  const int QS = D + 4;                          // row stride of qs and kv (floats)
  const int CR = f32_chunk_rows(D);
  // query heads h0 .. h0+7 rotated at t (fp64 angle), padding heads zero
  for (int x = tid; x < kF32Heads * D; x += kF32Threads) {
    const int hh = x / D, d = x % D;
    qs[hh * QS + d] = (h0 + hh < H) ? q[(int64_t)(h0 + hh) * D + d] : 0.f;
    run[x] = 0.f;
    tot[x] = 0.f;
  }
  if (tid < kF32Heads) { m_r[tid] = -INFINITY; l_r[tid] = 0.f; m_tot[tid] = -INFINITY; l_tot[tid] = 0.f; }
  __syncthreads();
  for (int x = tid; x < kF32Heads * (R / 2); x += kF32Threads) {
    const int hh = x / (R / 2), p = x % (R / 2);
    rope_pair(qs[hh * QS + D - R + 2 * p], qs[hh * QS + D - R + 2 * p + 1], L.theta()[p], g.t);
  }
  __syncthreads();
  // rows [r0, r0 + CR) of the tile to kv (coalesced 16-byte loads; no row: zeros)
  auto stage = [&](int r0) {
    const int D4 = D / 4;
    for (int x = tid; x < CR * D4; x += kF32Threads) {
      const int rr = x / D4, c4 = x % D4;
      const float* src = r0 + rr < kTileRows ? rows[r0 + rr] : nullptr;
      *reinterpret_cast<float4*>(kv + rr * QS + 4 * c4) =
          src != nullptr ? reinterpret_cast<const float4*>(src)[c4] : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };

  bool chunk_has = false;                        // the current chunk holds a tile with rows
  // two-level fold: the finished chunk's (m, l, O) into the total (an empty
  // chunk is skipped, as the fold kernel skips its partial); the chunk
  // result starts again empty
  auto fold_chunk = [&]() {
    if (chunk_has) {
      if (tid < kF32Heads) {
        float mn, al, be;
        fold_coef(m_tot[tid], m_r[tid], mn, al, be);
        alpha[tid] = al;
        beta[tid] = be;
        m_tot[tid] = mn;
        l_tot[tid] = fold_val(l_tot[tid], al, l_r[tid], be);
      }
      __syncthreads();
      for (int x = tid; x < kF32Heads * D; x += kF32Threads) {
        const int hh = x / D;
        tot[x] = fold_val(tot[x], alpha[hh], run[x], beta[hh]);
      }
      __syncthreads();
    }
    if (tid < kF32Heads) { m_r[tid] = -INFINITY; l_r[tid] = 0.f; }
    chunk_has = false;
    __syncthreads();
  };

  for (int tt = tt0; tt < tt_end; ++tt) {
    if (two_level && tt > tt0 && tt % g.chunk == 0) fold_chunk();
    int any = 0;
    if (tid < kTileRows) {
      rows[tid] = f32_row(a, g, i, tt, tid);
      any = rows[tid] != nullptr;
    }
    if (__syncthreads_count(any) == 0) continue;   // a tile without rows
    chunk_has = true;
    // logits from the staged rows: item (head hh, row r), d ascending
    for (int r0 = 0; r0 < kTileRows; r0 += CR) {
      stage(r0);
      __syncthreads();
      for (int x = tid; x < kF32Heads * CR; x += kF32Threads) {
        const int hh = x % kF32Heads, rr = x / kF32Heads, r = r0 + rr;
        float u = -INFINITY;
        if (r < kTileRows && rows[r] != nullptr) {
          const float* qh = qs + hh * QS;
          const float* k = kv + rr * QS;
          float acc = 0.f;
          for (int d = 0; d < D; ++d) acc = fmaf(qh[d], k[d], acc);
          u = acc * a.scale;
        }
        if (r < kTileRows) us[hh * kTileRows + r] = u;
      }
      __syncthreads();
    }
    // per head: m_t = max, then p = e^{u - m_t} in place, l_t = sum (r ascending)
    if (tid < kF32Heads) {
      const float* uh = us + tid * kTileRows;
      float mx = -INFINITY;
      for (int r = 0; r < kTileRows; ++r) mx = fmaxf(mx, uh[r]);
      m_t[tid] = mx;
    }
    __syncthreads();
    for (int x = tid; x < kF32Heads * kTileRows; x += kF32Threads) {
      const int hh = x / kTileRows, r = x % kTileRows;
      us[x] = rows[r] != nullptr ? expf(us[x] - m_t[hh]) : 0.f;
    }
    __syncthreads();
    if (tid < kF32Heads) {
      const float* uh = us + tid * kTileRows;
      float l = 0.f;
      for (int r = 0; r < kTileRows; ++r) l += uh[r];
      l_t[tid] = l;
    }
    __syncthreads();
    // O_t[h][d] = sum over r ascending of p v[r][d], folded into the chunk's result
    if (tid < kF32Heads) {
      float mn, al, be;
      fold_coef(m_r[tid], m_t[tid], mn, al, be);
      alpha[tid] = al;
      beta[tid] = be;
      l_r[tid] = fold_val(l_r[tid], al, l_t[tid], be);
      m_r[tid] = mn;
    }
    __syncthreads();
    // O_t[h][d] = sum over r ascending of p v[r][d], from the staged rows;
    // thread tid owns the outputs x = tid + kF32Threads * e
    float o[kF32MaxOut];
#pragma unroll
    for (int e = 0; e < kF32MaxOut; ++e) o[e] = 0.f;
    for (int r0 = 0; r0 < kTileRows; r0 += CR) {
      stage(r0);
      __syncthreads();
      const int r1 = r0 + CR < kTileRows ? r0 + CR : kTileRows;
#pragma unroll
      for (int e = 0; e < kF32MaxOut; ++e) {
        const int x = tid + kF32Threads * e;
        if (x < kF32Heads * D) {
          const int hh = x / D, d = x % D;
          const float* ph = us + hh * kTileRows;
          for (int r = r0; r < r1; ++r)
            if (rows[r] != nullptr) o[e] = fmaf(ph[r], kv[(r - r0) * QS + d], o[e]);
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int e = 0; e < kF32MaxOut; ++e) {
      const int x = tid + kF32Threads * e;
      if (x >= kF32Heads * D) continue;
      const int hh = x / D;
      run[x] = fold_val(run[x], alpha[hh], o[e], beta[hh]);
    }
    __syncthreads();
  }
  if (kSplit) {
    // the chunk's result (or an empty partial) to the workspace; a chunk of
    // one tile holds that tile's partial exactly
    const int64_t slot = (int64_t)i * a.chunks_max + c0;
    if (tid < kF32Heads && h0 + tid < H)
      a.ws_ml[slot * H + h0 + tid] = chunk_has ? make_float2(m_r[tid], l_r[tid]) : make_float2(-INFINITY, 0.f);
    if (chunk_has)
      for (int x = tid; x < kF32Heads * D; x += kF32Threads) {
        const int hh = x / D, d = x % D;
        if (h0 + hh < H) a.ws_o[(slot * H + h0 + hh) * D + d] = run[x];
      }
    return;
  }
  if (two_level) fold_chunk();
  const float* res = two_level ? tot : run;
  const float* m_res = two_level ? m_tot : m_r;
  const float* l_res = two_level ? l_tot : l_r;
  // out = O e^{m - mu} / (l e^{m - mu} + e^{sink - mu})
  if (tid < kF32Heads) {
    float cm, dn;
    finish_coef(m_res[tid], h0 + tid < H ? a.sink[h0 + tid] : 0.f, l_res[tid], cm, dn);
    alpha[tid] = cm;
    beta[tid] = dn;
  }
  __syncthreads();
  float* out = static_cast<float*>(a.out) + (int64_t)i * H * D;
  for (int x = tid; x < kF32Heads * D; x += kF32Threads) {
    const int hh = x / D, d = x % D;
    if (h0 + hh < H) out[(int64_t)(h0 + hh) * D + d] = finish_f32(res[x], alpha[hh], beta[hh]);
  }
}

cudaError_t launch_attn_f32(const Layout& L, int layer, int n, const int32_t* req_ids, const float* q,
                            const int32_t* topk, int k, const float* sink, float scale, float* out, void* ws,
                            cudaStream_t st, int q_per_req, const char* win_snap) {
  const size_t sm = (size_t)f32_smem(L.D).total;
  AttnArgs a{L, layer, n, req_ids, q, topk, k, sink, scale, out, kF32Heads, nullptr, nullptr, 0, 1, 0,
             q_per_req, win_snap};
  const int n_hg = (L.H + kF32Heads - 1) / kF32Heads;
  if (ws == nullptr) {
    cudaError_t e = cudaFuncSetAttribute(attn_f32_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    attn_f32_kernel<false><<<dim3(n, n_hg), kF32Threads, sm, st>>>(a);
    note_launch();
    return cudaGetLastError();
  }
  a.chunks_max = attn_chunks_max(L, layer, k);
  a.ws_o = static_cast<float*>(ws);
  a.ws_ml = reinterpret_cast<float2*>(static_cast<char*>(ws) + (int64_t)n * a.chunks_max * L.H * L.D * 4);
  cudaError_t e = cudaFuncSetAttribute(attn_f32_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  attn_f32_kernel<true><<<dim3(a.chunks_max, n_hg, n), kF32Threads, sm, st>>>(a);
  note_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attn_fold(a, st);
}

}  // namespace csa
