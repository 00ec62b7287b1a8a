// Lightning-indexer scores on CUDA cores (csa_index_scores, reference launch).
//
// Page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力": the query's index
// heads are scored against the compressed index keys after a ReLU; podcast
// summary page, section "2.1 推理与计算效率": the indexer path runs in FP4.
// Score of key j: s_j = sum_h w_h * max(0, q^_h . k^_j), q^ and k^ MXFP4.
//
// Arithmetic (fixed, shared by every launch shape): for each head the dot
// product is accumulated per 32-value block as an exact fp32 sum of E2M1
// products (all are multiples of 1/4 below 2^12), scaled by the two blocks'
// E8M0 scales (exact), and the block results are added in block order; the
// heads are then combined in head order with fp32 fma.  One thread owns one
// key, so the reduction order never depends on the launch shape.
#include "common.cuh"

namespace csa {

struct IndexArgs {
  Layout L;
  int layer;
  int n;
  const int32_t* req_ids;
  const float* q_idx;
  const float* w;
  float* scores;
  int64_t ld;
  int32_t* n_valid;
  int tiles_per_cta;   // 128-key tiles handled by one CTA (launch shape only)
};

constexpr int kMaxHI = 64;
constexpr int kMaxDI = 128;

__global__ void __launch_bounds__(128) index_simt_kernel(IndexArgs a) {
  __shared__ float qv[kMaxHI][kMaxDI];     // E2M1 values of the quantised query
  __shared__ int qe[kMaxHI][kMaxDI / 32];  // its E8M0 exponents (unbiased)
  __shared__ float ws[kMaxHI];
  const Layout& L = a.L;
  const int HI = L.HI, dI = L.dI, CH = dI / 32;
  const int i = blockIdx.y;
  const int req = a.req_ids[i];
  if (req < 0 || req >= L.max_req) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_err(L, kErrBounds, i);
    return;
  }
  const int64_t T = L.lengths()[(int64_t)a.layer * L.max_req + req];
  const int64_t N = T / kCsaM;
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    a.n_valid[i] = (int32_t)N;
    if (N > a.ld) set_err(L, kErrLd, i);
  }
  if (N > a.ld) return;
  const int64_t first_tile = (int64_t)blockIdx.x * a.tiles_per_cta;
  if (first_tile * 128 >= N) return;
  // quantise this query's index heads to MXFP4 (same rule as the keys)
  const float* q = a.q_idx + (int64_t)i * HI * dI;
  const int wid = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int blk = wid; blk < HI * CH; blk += 4) {
    const int h = blk / CH, c = blk % CH;
    const float x = q[h * dI + c * 32 + lane];
    float am = fabsf(x);
    for (int o = 16; o > 0; o >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, o));
    const int e = mx_exponent(am);
    const float y = scale_pow2(x, e);
    const float y1 = __shfl_xor_sync(0xffffffffu, y, 1);
    const uint8_t b = (lane & 1) ? e2m1x2_rn(y1, y) : e2m1x2_rn(y, y1);
    qv[h][c * 32 + lane] = e2m1_val((lane & 1) ? (b >> 4) : (b & 15));
    if (lane == 0) qe[h][c] = e;
  }
  for (int h = threadIdx.x; h < HI; h += blockDim.x) ws[h] = a.w[(int64_t)i * HI + h];
  __syncthreads();
  const int32_t* bt = L.block_table(req);
  for (int64_t tile = first_tile; tile < first_tile + a.tiles_per_cta; ++tile) {
    const int64_t j = tile * 128 + threadIdx.x;
    if (j >= N) break;
    const int32_t blk = bt[j / kCsaPerBlock];
    const int s = (int)(j % kCsaPerBlock);
    const char* bp = L.block(blk, a.layer);
    const uint8_t* codes = reinterpret_cast<const uint8_t*>(bp + L.blk_idx_codes);
    const uint8_t* scl = reinterpret_cast<const uint8_t*>(bp + L.blk_idx_scale) + s * CH;
    float dot[kMaxHI];
#pragma unroll
    for (int h = 0; h < kMaxHI; ++h) dot[h] = 0.f;
    for (int c = 0; c < CH; ++c) {
      const uint4 raw = *reinterpret_cast<const uint4*>(codes + (s >> 3) * (CH * 128) + c * 128 + (s & 7) * 16);
      const uint32_t wds[4] = {raw.x, raw.y, raw.z, raw.w};
      float kv[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) kv[t] = e2m1_val((wds[t >> 3] >> ((t & 7) * 4)) & 15u);
      const int ek = (int)scl[c] - 127;
#pragma unroll 4
      for (int h = 0; h < kMaxHI; ++h) {
        if (h < HI) {
          float acc = 0.f;
#pragma unroll
          for (int t = 0; t < 32; ++t) acc = fmaf(qv[h][c * 32 + t], kv[t], acc);
          dot[h] += ldexpf(acc, ek + qe[h][c]);   // exact: acc * 2^e
        }
      }
    }
    float sc = 0.f;
#pragma unroll
    for (int h = 0; h < kMaxHI; ++h)
      if (h < HI) sc = fmaf(ws[h], fmaxf(dot[h], 0.f), sc);
    a.scores[(int64_t)i * a.ld + j] = sc;
  }
}

cudaError_t launch_index_simt(const Layout& L, int layer, int n, const int32_t* req_ids,
                              const float* q_idx, const float* w, float* scores, int64_t ld,
                              int32_t* n_valid, int tiles_per_cta, cudaStream_t st) {
  IndexArgs a{L, layer, n, req_ids, q_idx, w, scores, ld, n_valid, tiles_per_cta};
  const int64_t tiles = (ld + 127) / 128;
  const int64_t ctas = tiles > 0 ? (tiles + tiles_per_cta - 1) / tiles_per_cta : 1;
  dim3 grid((unsigned)ctas, (unsigned)n);
  index_simt_kernel<<<grid, 128, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace csa
