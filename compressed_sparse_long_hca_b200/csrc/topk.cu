// Top-k selector (csa_topk).
//
// Page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力": the top-k
// selector keeps the 512 (Flash) or 1024 (Pro) best-scoring compressed
// entries.  Selection rule (fixed here): the k largest scores, equal scores
// going to the lower index, -0.0 == +0.0, output ascending, -1 padding.
//
// Method: an exact radix select on order-preserving 32-bit keys.  Four 8-bit
// passes of shared-memory histograms narrow the k-th largest key to one value
// T and give the number of ties at T that still fit; a final ordered pass
// emits every index with key > T and the first `ties` indices with key == T,
// in ascending order, through block-wide prefix sums.  Integer histograms and
// ordered prefix sums make the result independent of thread scheduling.
#include "common.cuh"

namespace csa {

__device__ __forceinline__ uint32_t order_key(float s) {
  const uint32_t b = __float_as_uint(s + 0.0f);       // -0.0 -> +0.0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

struct TopkArgs {
  const float* scores;
  int64_t ld;
  const int32_t* n_valid;
  int n;
  int k;
  int32_t* out;
  int32_t* err;   // device error word (may be null)
};

// Exclusive block prefix sum of `v` (blockDim.x == 1024); also returns the total.
__device__ __forceinline__ int block_excl_scan(int v, int* wsum, int& total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[w] = x;
  __syncthreads();
  if (w == 0) {
    int s = wsum[lane];
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, s, o);
      if (lane >= o) s += y;
    }
    wsum[lane] = s;   // inclusive over warps
  }
  __syncthreads();
  total = wsum[31];
  const int before = (w > 0 ? wsum[w - 1] : 0) + x - v;
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(1024) topk_radix_kernel(TopkArgs a) {
  __shared__ int hist[256];
  __shared__ int wsum[32];
  __shared__ uint32_t s_prefix, s_mask;
  __shared__ int s_remaining;
  const int i = blockIdx.x;
  const float* s = a.scores + (int64_t)i * a.ld;
  int32_t* out = a.out + (int64_t)i * a.k;
  int64_t N = a.n_valid[i];
  if (N < 0 || N > a.ld) {
    if (threadIdx.x == 0 && a.err) {
      if (atomicCAS(a.err, 0, (int32_t)kErrLd) == 0) a.err[1] = i;
    }
    N = 0;
  }
  const int k = a.k;
  if (N <= k) {
    for (int64_t j = threadIdx.x; j < k; j += blockDim.x) out[j] = j < N ? (int32_t)j : -1;
    return;
  }
  if (threadIdx.x == 0) { s_prefix = 0; s_mask = 0; s_remaining = k; }
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    const uint32_t prefix = s_prefix, mask = s_mask;
    for (int64_t j = threadIdx.x; j < N; j += blockDim.x) {
      const uint32_t key = order_key(s[j]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFF], 1);
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      int rem = s_remaining;
      int d = 255;
      for (; d > 0; --d) {
        if (hist[d] >= rem) break;
        rem -= hist[d];
      }
      s_remaining = rem;
      s_prefix = prefix | ((uint32_t)d << shift);
      s_mask = mask | (0xFFu << shift);
    }
    __syncthreads();
  }
  const uint32_t T = s_prefix;
  const int ties = s_remaining;        // indices with key == T still to take
  int sel_base = 0, eq_base = 0;
  for (int64_t j0 = 0; j0 < N; j0 += blockDim.x) {
    const int64_t j = j0 + threadIdx.x;
    uint32_t key = 0;
    if (j < N) key = order_key(s[j]);
    const int eq = (j < N && key == T) ? 1 : 0;
    int eq_total;
    const int eq_before = block_excl_scan(eq, wsum, eq_total);
    const int take = (j < N) && (key > T || (eq && eq_base + eq_before < ties)) ? 1 : 0;
    int sel_total;
    const int pos = block_excl_scan(take, wsum, sel_total);
    if (take) out[sel_base + pos] = (int32_t)j;
    sel_base += sel_total;
    eq_base += eq_total;
  }
}

cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* n_valid, int n, int k,
                        int32_t* out, int32_t* err, cudaStream_t st) {
  TopkArgs a{scores, ld, n_valid, n, k, out, err};
  topk_radix_kernel<<<n, 1024, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace csa
