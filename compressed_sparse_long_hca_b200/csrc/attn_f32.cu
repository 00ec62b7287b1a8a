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
// (m_t, l_t, O_t), folded in tile order with the shared fold arithmetic, the
// sink last.  Inside a tile every sum runs in a fixed order:
//   u[h][r]  = scale * (sum over d ascending of q[h][d] k[r][d])
//   l_t[h]   = sum over r ascending of e^{u - m_t}
//   O_t[h][d] = sum over r ascending of e^{u - m_t} v[r][d]
// so that a head's result depends on nothing but the query.  Launch variants:
//   * whole-query launch: one CTA per (query, head group) walks the tiles and
//     folds each into a running result in shared memory;
//   * split launch: one CTA per (query, head group, tile) writes its partial
//     to the workspace, and the shared fold kernel folds them.
// Both give identical bits.
#include "attn_common.cuh"
#include "common.cuh"

namespace csa {

namespace {

constexpr int kF32Threads = 256;
constexpr int kF32Heads = 8;        // heads per CTA

struct F32Smem {
  int64_t q, u, rows, run, stats, total;
};

__host__ __device__ inline F32Smem f32_smem(int D) {
  F32Smem s{};
  int64_t o = 0;
  s.q = o;     o += (int64_t)kF32Heads * D * 4;            // rotated query heads
  s.u = o;     o += (int64_t)kF32Heads * kTileRows * 4;    // logits, then e^{u - m_t}
  s.rows = o;  o += (int64_t)kTileRows * 8;                // row addresses (null = no row)
  s.run = o;   o += (int64_t)kF32Heads * D * 4;            // running O (whole-query launch)
  s.stats = o; o += (int64_t)6 * kF32Heads * 4;            // m_t, l_t, m, l, alpha, beta
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
  if (rr < g.total) return L.ring_row_f32(g.req, a.layer, (int)((g.w0 + (rr - g.n_list)) % kWindow));
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
  float* m_t = reinterpret_cast<float*>(smem_raw + S.stats);
  float* l_t = m_t + kF32Heads;
  float* m_r = l_t + kF32Heads;
  float* l_r = m_r + kF32Heads;
  float* alpha = l_r + kF32Heads;
  float* beta = alpha + kF32Heads;
  const int tid = threadIdx.x;
  const int i = kSplit ? (int)blockIdx.z : (int)blockIdx.x;
  const int h0 = blockIdx.y * kF32Heads;
  const int tt0 = kSplit ? (int)blockIdx.x : 0;
  QueryGeom g;
  const bool reporter = tid == 0 && blockIdx.y == 0 && (!kSplit || blockIdx.x == 0);
  if (!query_geom(a, i, g, reporter)) return;
  if (kSplit) {
    if (g.n_tiles > a.tiles_max) {
      if (reporter) set_err(L, kErrBounds, 4000000 + i);
      return;
    }
    if (tt0 >= g.n_tiles) return;
  }
  const int tt_end = kSplit ? tt0 + 1 : g.n_tiles;
  const float* q = static_cast<const float*>(a.q) + ((int64_t)i * H) * D;

  // query heads h0 .. h0+7 rotated at t (fp64 angle), padding heads zero
  for (int x = tid; x < kF32Heads * D; x += kF32Threads) {
    const int hh = x / D, d = x % D;
    qs[x] = (h0 + hh < H) ? q[(int64_t)(h0 + hh) * D + d] : 0.f;
    run[x] = 0.f;
  }
  if (tid < kF32Heads) { m_r[tid] = -INFINITY; l_r[tid] = 0.f; }
  __syncthreads();
  for (int x = tid; x < kF32Heads * (R / 2); x += kF32Threads) {
    const int hh = x / (R / 2), p = x % (R / 2);
    rope_pair(qs[hh * D + D - R + 2 * p], qs[hh * D + D - R + 2 * p + 1], L.theta()[p], g.t);
  }
  __syncthreads();

  for (int tt = tt0; tt < tt_end; ++tt) {
    int any = 0;
    if (tid < kTileRows) {
      rows[tid] = f32_row(a, g, i, tt, tid);
      any = rows[tid] != nullptr;
    }
    if (__syncthreads_count(any) == 0) {        // a tile without rows
      if (kSplit && tid < kF32Heads && h0 + tid < H)
        a.ws_ml[((int64_t)i * a.tiles_max + tt) * H + h0 + tid] = make_float2(-INFINITY, 0.f);
      continue;
    }
    // logits: thread (row r, heads hh, hh + 2, ...): d ascending
    for (int x = tid; x < kF32Heads * kTileRows; x += kF32Threads) {
      const int r = x % kTileRows, hh = x / kTileRows;
      const float* k = rows[r];
      float u = -INFINITY;
      if (k != nullptr) {
        const float* qh = qs + hh * D;
        float acc = 0.f;
        for (int d = 0; d < D; ++d) acc = fmaf(qh[d], k[d], acc);
        u = acc * a.scale;
      }
      us[hh * kTileRows + r] = u;
    }
    __syncthreads();
    // per head: m_t = max, then p = e^{u - m_t} in place, l_t = sum (r ascending)
    if (tid < kF32Heads) {
      float* uh = us + tid * kTileRows;
      float mx = -INFINITY;
      for (int r = 0; r < kTileRows; ++r) mx = fmaxf(mx, uh[r]);
      float l = 0.f;
      for (int r = 0; r < kTileRows; ++r) {
        const float p = rows[r] != nullptr ? expf(uh[r] - mx) : 0.f;
        uh[r] = p;
        l += p;
      }
      m_t[tid] = mx;
      l_t[tid] = l;
    }
    __syncthreads();
    // O_t[h][d] = sum over r ascending of p v[r][d]; fold or write out
    if (!kSplit && tid < kF32Heads) {
      float mn, al, be;
      fold_coef(m_r[tid], m_t[tid], mn, al, be);
      alpha[tid] = al;
      beta[tid] = be;
      l_r[tid] = fold_val(l_r[tid], al, l_t[tid], be);
      m_r[tid] = mn;
    }
    __syncthreads();
    for (int x = tid; x < kF32Heads * D; x += kF32Threads) {
      const int hh = x / D, d = x % D;
      const float* ph = us + hh * kTileRows;
      float o = 0.f;
      for (int r = 0; r < kTileRows; ++r)
        if (rows[r] != nullptr) o = fmaf(ph[r], rows[r][d], o);
      if (kSplit) {
        if (h0 + hh < H) a.ws_o[(((int64_t)i * a.tiles_max + tt) * H + h0 + hh) * D + d] = o;
      } else {
        run[x] = fold_val(run[x], alpha[hh], o, beta[hh]);
      }
    }
    if (kSplit && tid < kF32Heads && h0 + tid < H)
      a.ws_ml[((int64_t)i * a.tiles_max + tt) * H + h0 + tid] = make_float2(m_t[tid], l_t[tid]);
    __syncthreads();
  }
  if (!kSplit) {
    // out = O e^{m - mu} / (l e^{m - mu} + e^{sink - mu})
    if (tid < kF32Heads) {
      float cm, dn;
      finish_coef(m_r[tid], h0 + tid < H ? a.sink[h0 + tid] : 0.f, l_r[tid], cm, dn);
      alpha[tid] = cm;
      beta[tid] = dn;
    }
    __syncthreads();
    float* out = static_cast<float*>(a.out) + (int64_t)i * H * D;
    for (int x = tid; x < kF32Heads * D; x += kF32Threads) {
      const int hh = x / D, d = x % D;
      if (h0 + hh < H) out[(int64_t)(h0 + hh) * D + d] = finish_f32(run[x], alpha[hh], beta[hh]);
    }
  }
}

cudaError_t launch_attn_f32(const Layout& L, int layer, int n, const int32_t* req_ids, const float* q,
                            const int32_t* topk, int k, const float* sink, float scale, float* out, void* ws,
                            cudaStream_t st) {
  const size_t sm = (size_t)f32_smem(L.D).total;
  AttnArgs a{L, layer, n, req_ids, q, topk, k, sink, scale, out, kF32Heads, nullptr, nullptr, 0, 1};
  const int n_hg = (L.H + kF32Heads - 1) / kF32Heads;
  if (ws == nullptr) {
    cudaError_t e = cudaFuncSetAttribute(attn_f32_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    attn_f32_kernel<false><<<dim3(n, n_hg), kF32Threads, sm, st>>>(a);
    note_launch();
    return cudaGetLastError();
  }
  a.tiles_max = attn_tiles_max(L, layer, k);
  a.ws_o = static_cast<float*>(ws);
  a.ws_ml = reinterpret_cast<float2*>(static_cast<char*>(ws) + (int64_t)n * a.tiles_max * L.H * L.D * 4);
  cudaError_t e = cudaFuncSetAttribute(attn_f32_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  attn_f32_kernel<true><<<dim3(a.tiles_max, n_hg, n), kF32Threads, sm, st>>>(a);
  note_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_attn_fold(a, st);
}

}  // namespace csa
