// Multi-query decode attention on CUDA cores (csa_hca_decode_attn, reference
// launch).
//
// Page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力": the selected
// compressed entries and the sliding window's raw tokens are fed together to
// multi-query attention (all query heads share one KV head); section
// "HCA——重度压缩注意力": HCA attends densely to every compressed entry, both
// keep the latest 128 raw tokens, each head has a learnable sink logit added
// to the softmax denominator, RoPE acts on the last 64 dims only, and the
// stored KV is FP8 (non-RoPE dims) + BF16 (RoPE dims).
//
// Per query: rows = selected entries (ascending) then the window (ascending
// positions); K = V = the dequantised row.  Each warp owns one head and walks
// the rows in fixed tiles of 32 with an online softmax; the sink enters at the
// end.  The per-head arithmetic does not depend on how many heads share a
// thread block, so every launch shape returns identical bits, and no query's
// reduction is ever split across thread blocks.
#include "common.cuh"

namespace csa {

struct AttnArgs {
  Layout L;
  int layer;
  int n;
  const int32_t* req_ids;
  const uint16_t* q;
  const int32_t* topk;
  int k;
  const float* sink;
  float scale;
  uint16_t* out;
  int heads_per_cta;
};

constexpr int kTileRows = 32;

__global__ void __launch_bounds__(256) attn_simt_kernel(AttnArgs a) {
  extern __shared__ float sm[];
  const Layout& L = a.L;
  const int D = L.D, R = L.R, H = L.H;
  const int DP = D + 4;                        // padded row stride (bank spread)
  float* tile = sm;                            // [32][DP]
  float* qs = tile + kTileRows * DP;           // [heads_per_cta][D]
  const int i = blockIdx.x;
  const int h0 = blockIdx.y * a.heads_per_cta;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nthreads = blockDim.x;
  const int req = a.req_ids[i];
  if (req < 0 || req >= L.max_req) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_err(L, kErrBounds, i);
    return;
  }
  const bool csa = a.layer < L.n_csa;
  const int64_t T = L.lengths()[(int64_t)a.layer * L.max_req + req];
  if (T <= 0) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_err(L, kErrBounds, 1000000 + i);
    return;
  }
  const int64_t t = T - 1;                               // query position
  const int64_t n_entries = csa ? T / kCsaM : T / kHcaM;
  const int64_t w0 = t - (kWindow - 1) > 0 ? t - (kWindow - 1) : 0;
  const int64_t n_win = t - w0 + 1;
  const int32_t* sel = csa ? a.topk + (int64_t)i * a.k : nullptr;
  const int64_t n_sel = csa ? a.k : n_entries;           // list slots (CSA may hold -1)
  // rotate this CTA's query heads at position t (fp32 from the BF16 input)
  const uint16_t* qin = a.q + ((int64_t)i * H + h0) * D;
  for (int x = threadIdx.x; x < a.heads_per_cta * D; x += nthreads) qs[x] = bf16_val(qin[x]);
  __syncthreads();
  for (int x = threadIdx.x; x < a.heads_per_cta * (R / 2); x += nthreads) {
    const int hh = x / (R / 2), p = x % (R / 2);
    float* qh = qs + hh * D;
    rope_pair(qh[D - R + 2 * p], qh[D - R + 2 * p + 1], p, R, t, L.rope_base);
  }
  __syncthreads();
  const int my_h = warp;                       // head inside the CTA owned by this warp
  const bool active = my_h < a.heads_per_cta;
  const int DL = D / 32;                       // dims per lane
  float o[16];
#pragma unroll
  for (int x = 0; x < 16; ++x) o[x] = 0.f;
  float m = -INFINITY, l = 0.f;
  const char* st = L.state(req, a.layer);
  // walk the rows: list slots 0..n_sel-1, then window rows
  const int64_t total = n_sel + n_win;
  for (int64_t r0 = 0; r0 < total; r0 += kTileRows) {
    // dequantise the tile's rows into shared memory; invalid rows get a marker
    __shared__ int valid[kTileRows];
    for (int rr = warp; rr < kTileRows; rr += nthreads / 32) {
      const int64_t r = r0 + rr;
      const uint8_t* fp8 = nullptr;
      const uint16_t* bf = nullptr;
      const float* scp = nullptr;
      float sc = 0.f;
      bool ok = false;
      if (r < n_sel) {
        const int64_t j = csa ? (int64_t)sel[r] : r;
        if (j >= 0) {
          if (j >= n_entries) {
            if (lane == 0) set_err(L, kErrBounds, 2000000 + i);
          } else {
            L.entry_row(req, a.layer, j, &fp8, &bf, &scp);
            sc = *scp;
            ok = true;
          }
        }
      } else if (r < total) {
        const int slot = (int)((w0 + (r - n_sel)) % kWindow);
        fp8 = reinterpret_cast<const uint8_t*>(st + L.ring_fp8) + (int64_t)slot * (D - R);
        bf = reinterpret_cast<const uint16_t*>(st + L.ring_bf16) + (int64_t)slot * R;
        sc = reinterpret_cast<const float*>(st + L.ring_scale)[slot];
        ok = true;
      }
      float* dst = tile + rr * DP;
      if (ok) {
        for (int d = lane; d < D - R; d += 32) dst[d] = e4m3_val(fp8[d]) * sc;
        for (int d = lane; d < R; d += 32) dst[D - R + d] = bf16_val(bf[d]);
      }
      if (lane == 0) valid[rr] = ok ? 1 : 0;
    }
    __syncthreads();
    if (active) {
      const float* qh = qs + my_h * D;
      // logit of row `lane`
      float u = -INFINITY;
      if (valid[lane]) {
        const float* kr = tile + lane * DP;
        float acc = 0.f;
        for (int d = 0; d < D; ++d) acc = fmaf(qh[d], kr[d], acc);
        u = acc * a.scale;
      }
      float tmax = u;
      for (int off = 16; off > 0; off >>= 1) tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, off));
      if (tmax > -INFINITY) {
        const float mn = fmaxf(m, tmax);
        const float corr = expf(m - mn);       // 0 when m == -inf
        const float p = valid[lane] ? expf(u - mn) : 0.f;
        float ps = p;
        for (int off = 16; off > 0; off >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, off);
        l = l * corr + ps;
#pragma unroll
        for (int x = 0; x < 16; ++x) if (x < DL) o[x] *= corr;
        for (int rr = 0; rr < kTileRows; ++rr) {
          const float pr = __shfl_sync(0xffffffffu, p, rr);
          if (pr != 0.f) {
            const float* vr = tile + rr * DP;
#pragma unroll
            for (int x = 0; x < 16; ++x) if (x < DL) o[x] = fmaf(pr, vr[lane + 32 * x], o[x]);
          }
        }
        m = mn;
      }
    }
    __syncthreads();
  }
  if (active) {
    const int h = h0 + my_h;
    const float sk = a.sink[h];
    const float mf = fmaxf(m, sk);
    const float cm = expf(m - mf);
    const float den = l * cm + expf(sk - mf);
    uint16_t* dst = a.out + ((int64_t)i * H + h) * D;
#pragma unroll
    for (int x = 0; x < 16; ++x) if (x < DL) dst[lane + 32 * x] = bf16_rn(__fdiv_rn(o[x] * cm, den));
  }
}

cudaError_t launch_attn_simt(const Layout& L, int layer, int n, const int32_t* req_ids,
                             const uint16_t* q, const int32_t* topk, int k, const float* sink,
                             float scale, uint16_t* out, int heads_per_cta, cudaStream_t st) {
  AttnArgs a{L, layer, n, req_ids, q, topk, k, sink, scale, out, heads_per_cta};
  const size_t sm = ((size_t)kTileRows * (L.D + 4) + (size_t)heads_per_cta * L.D) * sizeof(float);
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(attn_simt_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 200 * 1024);
    attr_set = true;
  }
  dim3 grid(n, L.H / heads_per_cta);
  attn_simt_kernel<<<grid, 32 * (heads_per_cta < 8 ? 8 : heads_per_cta), sm, st>>>(a);
  return cudaGetLastError();
}

}  // namespace csa
