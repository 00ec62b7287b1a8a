// Lightning-indexer scores for caches in the fp32 storage format
// (csa_index_scores on a CSA_FMT_F32 cache), on the CUDA cores.
//
// Page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力": the query's
// index heads are scored against every compressed index key after a ReLU,
//   s_j = sum_h w_h * max(0, q_h . k_j),
// here with q and the stored keys in fp32 (no FP4 quantisation).  One thread
// computes one key's score in a fixed order (d ascending inside a head, heads
// ascending), so a score never depends on the grid, the batch or the launch
// variant; the two variants only differ in how many CTAs share a query.
#include "common.cuh"

namespace csa {

namespace {

constexpr int kIdxF32Threads = 256;

struct IndexF32Args {
  Layout L;
  int layer;
  int n;
  const int32_t* req_ids;
  const float* q_idx;     // [n][H_I][d_I]
  const float* w;         // [n][H_I]
  float* scores;          // [n][ld]
  int64_t ld;
  int32_t* n_valid;
  int q_per_req;          // 0: decode queries; C > 0: chunk queries (visible_tokens)
};

}  // namespace

// grid (CTAs per query, n); the CTAs of a query stride over its keys.
__global__ void __launch_bounds__(kIdxF32Threads) index_f32_kernel(IndexF32Args a) {
  extern __shared__ __align__(16) float sm_f[];
  const Layout& L = a.L;
  const int HI = L.HI, dI = L.dI;
  float* qs = sm_f;                 // [H_I][d_I]
  float* ws = sm_f + HI * dI;       // [H_I]
  const int i = blockIdx.y, tid = threadIdx.x;
  const int req = a.req_ids[i];
  if (req < 0 || req >= L.max_req) {
    if (blockIdx.x == 0 && tid == 0) {
      set_err(L, kErrBounds, i);
      a.n_valid[i] = 0;
    }
    return;
  }
  const int64_t T = visible_tokens(L.lengths()[(int64_t)a.layer * L.max_req + req], a.q_per_req, i);
  const int64_t N = T > 0 ? T / kCsaM : 0;
  if (blockIdx.x == 0 && tid == 0) {
    a.n_valid[i] = (int32_t)N;
    if (N > a.ld) set_err(L, kErrLd, i);
  }
  if (N > a.ld) return;
  for (int x = tid; x < HI * dI; x += kIdxF32Threads) qs[x] = a.q_idx[(int64_t)i * HI * dI + x];
  for (int x = tid; x < HI; x += kIdxF32Threads) ws[x] = a.w[(int64_t)i * HI + x];
  __syncthreads();
  float* out = a.scores + (int64_t)i * a.ld;
  for (int64_t j = (int64_t)blockIdx.x * kIdxF32Threads + tid; j < N; j += (int64_t)gridDim.x * kIdxF32Threads) {
    const float4* k4 = reinterpret_cast<const float4*>(L.index_key_f32(req, a.layer, j));
    float s = 0.f;
    for (int h = 0; h < HI; ++h) {
      const float* qh = qs + h * dI;
      float dot = 0.f;
      // 32 values of the key at a time, their loads in flight together (the
      // first head brings the key into L1 for the others); d ascending
      for (int d0 = 0; d0 < dI; d0 += 32) {
        float kv[32];
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const float4 v = k4[d0 / 4 + x];
          kv[4 * x] = v.x; kv[4 * x + 1] = v.y; kv[4 * x + 2] = v.z; kv[4 * x + 3] = v.w;
        }
#pragma unroll
        for (int d = 0; d < 32; ++d) dot = fmaf(qh[d0 + d], kv[d], dot);
      }
      s = fmaf(ws[h], fmaxf(dot, 0.f), s);
    }
    out[j] = s;
  }
}

cudaError_t launch_index_f32(const Layout& L, int layer, int n, const int32_t* req_ids, const float* q_idx,
                             const float* w, float* scores, int64_t ld, int32_t* n_valid, int ctas_per_query,
                             cudaStream_t st, int q_per_req) {
  IndexF32Args a{L, layer, n, req_ids, q_idx, w, scores, ld, n_valid, q_per_req};
  const size_t sm = (size_t)(L.HI * L.dI + L.HI) * 4;
  cudaError_t e = cudaFuncSetAttribute(index_f32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  index_f32_kernel<<<dim3(ctas_per_query, n), kIdxF32Threads, sm, st>>>(a);
  note_launch();
  return cudaGetLastError();
}

}  // namespace csa
