// Top-k selector (csa_topk).
//
// Page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力": the top-k
// selector keeps the 512 (Flash) or 1024 (Pro) best-scoring compressed
// entries.  Selection rule (fixed here): the k largest scores, equal scores
// going to the lower index, -0.0 == +0.0, output ascending, -1 padding.
//
// Method: an exact radix select on order-preserving 32-bit keys, run by one
// thread-block cluster per query.  Each CTA of the cluster owns a contiguous
// slice of the query's scores (kept in shared memory when it fits).  Three
// passes (11, 11 and 10 bits) build shared-memory histograms of the keys
// that still match the prefix found so far; the cluster adds its histograms
// through distributed shared memory and every CTA reads off the same digit.
// The passes end with the k-th largest key T and the number of ties at T
// that still fit.  The output pass exchanges per-CTA counts, so that each
// CTA writes its selected indices (all keys > T, then ties at T in index
// order) at the right place of the ascending list.  Integer histograms and
// ordered prefix sums make the result independent of thread scheduling and
// of the cluster's launch shape; the cluster barriers are hardware barriers,
// no thread spins on memory.
#include <cooperative_groups.h>

#include "common.cuh"

namespace cg = cooperative_groups;

namespace csa {

namespace {

constexpr int kTopkThreads = 1024;
constexpr int kBins = 2048;                // 11-bit digits
constexpr int kMaxCluster = 8;

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
  int32_t* err;          // device error word (may be null)
  int cache_keys;        // slices fit in shared memory
  int64_t slice_cap;     // keys per CTA slice buffer
};

// Exclusive block-wide prefix sum over kTopkThreads threads; returns the total.
__device__ __forceinline__ int block_excl_scan(int v, int* wsum, int* total) {
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
    wsum[lane] = s;
  }
  __syncthreads();
  *total = wsum[31];
  const int before = (w > 0 ? wsum[w - 1] : 0) + x - v;
  __syncthreads();
  return before;
}

struct TopkShared {
  int hist[kBins];          // this CTA's histogram
  int slice_sum[kBins];     // reduce-scatter: summed bins owned by this CTA
  int full[kBins];          // the cluster's summed histogram
  int wsum[32];
  int cnt[2];               // this CTA's (count > T, count == T)
  uint32_t digit;
  int remaining;
};

}  // namespace

template <int C>
__global__ void __cluster_dims__(C, 1, 1) __launch_bounds__(kTopkThreads, 1) topk_cluster_kernel(TopkArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + sizeof(TopkShared));
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int i = blockIdx.y;
  const int tid = threadIdx.x;
  const float* s = a.scores + (int64_t)i * a.ld;
  int32_t* out = a.out + (int64_t)i * a.k;
  int64_t N = a.n_valid[i];
  if (N < 0 || N > a.ld) {
    if (rank == 0 && tid == 0 && a.err) {
      if (atomicCAS(a.err, 0, (int32_t)kErrLd) == 0) a.err[1] = i;
    }
    N = 0;
  }
  const int k = a.k;
  if (N <= k) {   // every entry is selected: indices in order, then -1
    for (int64_t j = (int64_t)rank * kTopkThreads + tid; j < k; j += (int64_t)C * kTopkThreads)
      out[j] = j < N ? (int32_t)j : -1;
    return;       // uniform for the whole cluster (N is the cluster's)
  }
  const int64_t chunk = (N + C - 1) / C;
  const int64_t lo = (int64_t)rank * chunk;
  const int64_t hi = lo + chunk < N ? lo + chunk : N;
  const int64_t len = hi > lo ? hi - lo : 0;
  auto key_at = [&](int64_t x) -> uint32_t { return a.cache_keys ? keys[x] : order_key(s[lo + x]); };
  if (a.cache_keys) {
    // eight loads in flight per thread before any of them is used
    for (int64_t x0 = tid; x0 < len; x0 += 8 * kTopkThreads) {
      float v[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t x = x0 + (int64_t)u * kTopkThreads;
        v[u] = x < len ? s[lo + x] : 0.f;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t x = x0 + (int64_t)u * kTopkThreads;
        if (x < len) keys[x] = order_key(v[u]);
      }
    }
  }
  if (tid == 0) { sh.digit = 0; sh.remaining = k; }
  uint32_t prefix = 0;
  int remaining = k;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int p = 0; p < 3; ++p) {
    const int shift = shifts[p], width = widths[p];
    const uint32_t mask = (1u << width) - 1;
    for (int b = tid; b < kBins; b += kTopkThreads) sh.hist[b] = 0;
    __syncthreads();
    // lanes that hit the same bin add once (score distributions pile up in a
    // few top-bit bins, where per-lane atomics would serialise)
    for (int64_t x0 = tid - (tid & 31); x0 < len; x0 += kTopkThreads) {
      const int64_t x = x0 + (tid & 31);
      const uint32_t key = x < len ? key_at(x) : 0u;
      const bool hit = x < len && (p == 0 || (key >> (shift + width)) == prefix);
      const uint32_t bin = hit ? (key >> shift) & mask : 0xFFFFFFFFu;
      if (!__any_sync(0xffffffffu, hit)) continue;
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (hit && (tid & 31) == __ffs(peers) - 1) atomicAdd(&sh.hist[bin], __popc(peers));
    }
    // cluster reduce-scatter: CTA r sums bins [r*kBins/C, (r+1)*kBins/C)
    cluster.sync();
    constexpr int per = kBins / C;
    for (int b = tid; b < per; b += kTopkThreads) {
      int t = 0;
      for (int r = 0; r < C; ++r) t += cluster.map_shared_rank(&sh.hist[0], r)[rank * per + b];
      sh.slice_sum[b] = t;
    }
    cluster.sync();
    for (int b = tid; b < kBins; b += kTopkThreads)
      sh.full[b] = cluster.map_shared_rank(&sh.slice_sum[0], b / per)[b % per];
    __syncthreads();
    // digit d: the largest d with (count of digits > d) < remaining <= (count of digits >= d)
    {
      // suffix sums over bins, 2 bins per thread (kBins = 2 * kTopkThreads)
      const int b0 = kBins - 2 - 2 * tid;        // thread 0 owns the top bins
      const int c1 = sh.full[b0 + 1], c0 = sh.full[b0];
      int tot;
      const int before = block_excl_scan(c1 + c0, sh.wsum, &tot);   // counts of bins above b0 + 1
      if (before < remaining && before + c1 >= remaining) { sh.digit = (uint32_t)(b0 + 1); sh.remaining = remaining - before; }
      else if (before + c1 < remaining && before + c1 + c0 >= remaining) {
        sh.digit = (uint32_t)b0;
        sh.remaining = remaining - before - c1;
      }
      __syncthreads();
    }
    prefix = (prefix << width) | sh.digit;
    remaining = sh.remaining;
    // the histogram buffers are read remotely until every CTA has its copy
    cluster.sync();
  }
  const uint32_t T = prefix;        // the k-th largest key
  const int ties_needed = remaining;
  // ---- output: each warp owns a contiguous sub-slice, walked 32 keys at a
  //      time (lane l reads key base + l: conflict-free), so that ballots
  //      give ordered positions.
  const int lane = tid & 31, wid = tid >> 5;
  constexpr int kWarps = kTopkThreads / 32;
  const int64_t per_w = ((len + kWarps - 1) / kWarps + 31) / 32 * 32;
  const int64_t w_lo = (int64_t)wid * per_w < len ? (int64_t)wid * per_w : len;
  const int64_t w_hi = w_lo + per_w < len ? w_lo + per_w : len;
  const unsigned lt_mask = (1u << lane) - 1u;
  int gt = 0, eq = 0;   // warp totals (uniform across the warp)
  for (int64_t x0 = w_lo; x0 < w_hi; x0 += 32) {
    const int64_t x = x0 + lane;
    const uint32_t key = x < w_hi ? key_at(x) : 0u;
    gt += __popc(__ballot_sync(0xffffffffu, x < w_hi && key > T));
    eq += __popc(__ballot_sync(0xffffffffu, x < w_hi && key == T));
  }
  int gt_tot, eq_tot;
  const int gt_before = __shfl_sync(0xffffffffu, block_excl_scan(lane == 0 ? gt : 0, sh.wsum, &gt_tot), 0);
  const int eq_before = __shfl_sync(0xffffffffu, block_excl_scan(lane == 0 ? eq : 0, sh.wsum, &eq_tot), 0);
  if (tid == 0) { sh.cnt[0] = gt_tot; sh.cnt[1] = eq_tot; }
  cluster.sync();
  int sel_before = 0, take_cta = 0;
  {
    int tb = 0;
    for (int r = 0; r < C; ++r) {
      const int* c = cluster.map_shared_rank(&sh.cnt[0], r);
      const int g = c[0], e = c[1];
      int take = ties_needed - tb;
      take = take < 0 ? 0 : (take > e ? e : take);
      if (r < rank) sel_before += g + take;
      if (r == rank) take_cta = take;
      tb += e;
    }
  }
  // ties this warp may take: those among the CTA's first take_cta ties
  int w_ties = take_cta - eq_before;
  w_ties = w_ties < 0 ? 0 : (w_ties > eq ? eq : w_ties);
  int tot_sel;
  const int w_pos0 = __shfl_sync(0xffffffffu, block_excl_scan(lane == 0 ? gt + w_ties : 0, sh.wsum, &tot_sel), 0);
  int pos = sel_before + w_pos0;
  int ties_seen = 0;
  for (int64_t x0 = w_lo; x0 < w_hi; x0 += 32) {
    const int64_t x = x0 + lane;
    const uint32_t key = x < w_hi ? key_at(x) : 0u;
    const bool is_eq = x < w_hi && key == T;
    const unsigned eqb = __ballot_sync(0xffffffffu, is_eq);
    const int tie_rank = ties_seen + __popc(eqb & lt_mask);
    const bool take = x < w_hi && (key > T || (is_eq && tie_rank < w_ties));
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) out[pos + __popc(tb & lt_mask)] = (int32_t)(lo + x);
    pos += __popc(tb);
    ties_seen += __popc(eqb);
  }
  (void)gt_before;
  // no CTA may leave while others still read its shared memory
  cluster.sync();
}

cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* n_valid, int n, int k,
                        int32_t* out, int32_t* err, int cluster, cudaStream_t st) {
  if (n > 65535) return cudaErrorInvalidValue;
  const int64_t slice = (ld + cluster - 1) / cluster;
  const size_t base = sizeof(TopkShared);
  const size_t cap = 200 * 1024;
  const bool cache = base + (size_t)slice * 4 <= cap;
  const size_t sm = cache ? base + (size_t)slice * 4 : base;
  TopkArgs a{scores, ld, n_valid, n, k, out, err, cache ? 1 : 0, slice};
  dim3 grid(cluster, n);
  cudaError_t e;
  if (cluster == 8) {
    e = cudaFuncSetAttribute(topk_cluster_kernel<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cap);
    if (e != cudaSuccess) return e;
    topk_cluster_kernel<8><<<grid, kTopkThreads, sm, st>>>(a);
    note_launch();
  } else if (cluster == 4) {
    e = cudaFuncSetAttribute(topk_cluster_kernel<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)cap);
    if (e != cudaSuccess) return e;
    topk_cluster_kernel<4><<<grid, kTopkThreads, sm, st>>>(a);
    note_launch();
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace csa
