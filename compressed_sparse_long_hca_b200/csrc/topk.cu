// Top-k selector (csa_topk).
//
// Page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力": the top-k
// selector keeps the 512 (Flash) or 1024 (Pro) best-scoring compressed
// entries.  Selection rule (fixed here): the k largest scores, equal scores
// going to the lower index, -0.0 == +0.0, output ascending, -1 padding.
//
// Scores become order-preserving 32-bit keys.  One thread-block cluster per
// query; each CTA owns a contiguous slice of the query's keys, which one bulk
// copy brings into shared memory when it fits.
//
// Filter path (the usual case).
//   1. Threshold.  Every CTA reads the same sample of S keys (64 evenly
//      spaced runs of 64 consecutive keys) and
//      takes tau = the sample's r-th largest key, r chosen so that with
//      overwhelming probability fewer than r sampled keys lie above the
//      query's k-th key; then every key of the top k is >= tau, and about
//      r N / S keys pass, whatever the scores' distribution.  (Correctness
//      never depends on the sample: step 3 checks that at least k keys pass.)
//   2. Filter.  Each CTA counts its keys >= tau (warp ballots), the cluster
//      exchanges the counts through distributed shared memory, and each CTA
//      writes its passing (key, index) pairs, in index order, into the leader
//      CTA's candidate list at its offset.
//   3. Select.  If between k and kCandCap keys passed, the leader finds the
//      k-th largest candidate key T: one histogram of the candidates over
//      2048 equal bins of [tau, max] finds T's bin, and the few keys in that
//      bin are ranked against each other.  It then writes, in index order,
//      every candidate > T and the first k - #(> T) candidates == T.
// Radix path (when the filter does not apply, e.g. a tie class larger than
// kCandCap): an exact three-pass radix select (11, 11, 10 bits) with
// cluster-summed histograms, then an ordered output walk over the slices.
// Both paths are exact, so they return the same indices; integer counts and
// ordered prefix sums make the result independent of scheduling and of the
// cluster's size.  Cluster barriers are hardware barriers; the one wait on
// memory (the bulk copy's mbarrier) gives up after a time limit.
#include <cooperative_groups.h>

#include <mutex>

#include "common.cuh"
#include "tc.cuh"

namespace cg = cooperative_groups;

namespace csa {

namespace {

constexpr int kTopkThreads = 1024;
constexpr int kWarps = kTopkThreads / 32;
constexpr int kBins = 2048;                // 11-bit digits
constexpr int kSample = 4096;              // sampled keys for the threshold
constexpr int kSamplePer = kSample / kTopkThreads;
constexpr int kCandCap = 8192;             // candidate list capacity
constexpr int kCandPer = kCandCap / kTopkThreads;

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
  int cache_keys;        // every CTA's slice fits in shared memory
};

struct RadixBufs {
  int hist[kBins];          // this CTA's histogram
  int slice_sum[kBins];     // summed bins owned by this CTA
  int full[kBins];          // the cluster's summed histogram
};

struct TopkShared {
  union {
    uint2 cand[kCandCap];   // filter path (leader): (key, index) of the candidates, index order
    RadixBufs rx;           // radix path
  } u;
  int sel_hist[kBins];      // histogram of block_select
  uint32_t list[kTopkThreads];  // block_select: the keys of one bin
  int wsum[32];
  int scan_a[32], scan_b[32];   // warp totals of the one-barrier scans (one buffer per call site)
  int selw[2][32];          // block_select: warp totals of a round (alternating rounds)
  uint32_t mm[2][2][32];    // per-warp min / max (one buffer per call site)
  int cnt[2];               // radix path: this CTA's (count > T, count == T)
  int n_cand;               // filter path: this CTA's keys >= tau
  int n_list;
  int bin_count;
  uint32_t digit;
  int remaining;
  uint64_t bar;             // bulk copy of the slice
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

// Exclusive block-wide prefix sum with one barrier: warp scans, warp totals
// through `buf`.  A later call must not reuse `buf` before another barrier.
__device__ __forceinline__ int block_scan1(int v, int* buf, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) buf[w] = x;
  __syncthreads();
  const int tw = lane < kWarps ? buf[lane] : 0;
  *total = __reduce_add_sync(0xffffffffu, tw);
  return __reduce_add_sync(0xffffffffu, lane < w ? tw : 0) + x - v;
}

// Block-wide (min, max) of E keys per thread (flags mark the valid ones);
// one barrier (each call site has its own buffer).
template <int E>
__device__ __forceinline__ void block_minmax(const uint32_t (&v)[E], const bool (&ok)[E], uint32_t (*mm)[32],
                                             uint32_t* mn, uint32_t* mx) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  uint32_t a = 0xFFFFFFFFu, b = 0u;
#pragma unroll
  for (int e = 0; e < E; ++e)
    if (ok[e]) { a = min(a, v[e]); b = max(b, v[e]); }
  a = __reduce_min_sync(0xffffffffu, a);
  b = __reduce_max_sync(0xffffffffu, b);
  if (lane == 0) { mm[0][w] = a; mm[1][w] = b; }
  __syncthreads();
  *mn = __reduce_min_sync(0xffffffffu, mm[0][lane]);
  *mx = __reduce_max_sync(0xffffffffu, mm[1][lane]);
}

// The r-th largest of the valid keys (1 <= r <= #valid, every valid key in
// [kmin, kmax]), exactly: returns T and sets *ties = r - #{keys > T}.  Each
// round histograms the keys of the current range over up to 2048 equal
// bins and keeps the bin that holds the r-th key; once that bin holds at
// most kTopkThreads keys they are ranked against each other.  sh.sel_hist
// must be zero on entry and is zero again on return (each thread clears the
// bins it has read); sh.n_list likewise.
template <int E>
__device__ uint32_t block_select(const uint32_t (&v)[E], const bool (&ok)[E], int r, uint32_t kmin, uint32_t kmax,
                                 TopkShared& sh, int* ties) {
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  uint64_t base = kmin, width = (uint64_t)kmax - kmin + 1;
  int remaining = r;
  for (int round = 0;; ++round) {
    int shift = 0;
    while (((width - 1) >> shift) >= (uint64_t)kBins) ++shift;
#pragma unroll
    for (int e = 0; e < E; ++e)
      if (ok[e] && (uint64_t)v[e] >= base && (uint64_t)v[e] - base < width)
        atomicAdd(&sh.sel_hist[((uint64_t)v[e] - base) >> shift], 1);
    __syncthreads();
    {   // bin d: (count in bins > d) < remaining <= (count in bins >= d).  Warp w
        // owns bins 64w .. 64w+63, lane l the bins 64w+2l (c0) and 64w+2l+1 (c1).
      const int b0 = 64 * w + 2 * lane;
      const int c0 = sh.sel_hist[b0], c1 = sh.sel_hist[b0 + 1];
      sh.sel_hist[b0] = 0;
      sh.sel_hist[b0 + 1] = 0;
      int x = c0 + c1;                                 // suffix sum over lanes >= l
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_down_sync(0xffffffffu, x, o);
        if (lane + o < 32) x += y;
      }
      int* wt = sh.selw[round & 1];
      if (lane == 0) wt[w] = x;                        // warp total
      __syncthreads();
      const int tw = lane < kWarps ? wt[lane] : 0;
      const int before = __reduce_add_sync(0xffffffffu, lane > w ? tw : 0) + x - (c0 + c1);
      if (before < remaining && before + c1 >= remaining) {
        sh.digit = (uint32_t)(b0 + 1);
        sh.remaining = remaining - before;
        sh.bin_count = c1;
      } else if (before + c1 < remaining && before + c1 + c0 >= remaining) {
        sh.digit = (uint32_t)b0;
        sh.remaining = remaining - before - c1;
        sh.bin_count = c0;
      }
      __syncthreads();
    }
    const uint64_t d = sh.digit;
    const int in_bin = sh.bin_count;
    remaining = sh.remaining;
    base += d << shift;
    const uint64_t left = width - (d << shift);
    width = left < ((uint64_t)1 << shift) ? left : ((uint64_t)1 << shift);
    if (shift == 0) {
      *ties = remaining;
      return (uint32_t)base;
    }
    if (in_bin <= kTopkThreads) {   // rank the bin's keys against each other
#pragma unroll
      for (int e = 0; e < E; ++e)
        if (ok[e] && (uint64_t)v[e] >= base && (uint64_t)v[e] - base < width) sh.list[atomicAdd(&sh.n_list, 1)] = v[e];
      __syncthreads();
      const int m = sh.n_list;
      if (tid < m) {
        const uint32_t x = sh.list[tid];
        int gt = 0, ge = 0;
        for (int y = 0; y < m; ++y) {
          const uint32_t zz = sh.list[y];
          gt += zz > x ? 1 : 0;
          ge += zz >= x ? 1 : 0;
        }
        if (gt < remaining && remaining <= ge) {   // equal keys write equal values
          sh.digit = x;
          sh.remaining = remaining - gt;
        }
      }
      __syncthreads();
      *ties = sh.remaining;
      const uint32_t T = sh.digit;
      if (tid == 0) sh.n_list = 0;   // read above by every thread before the last barrier
      return T;
    }
  }
}

// Radix path: the k-th largest key of the query (all CTAs of the cluster)
// and how many keys equal to it are selected.
template <int C>
__device__ void radix_select(cg::cluster_group& cluster, TopkShared& sh, const float* s, int64_t lo, int64_t len,
                             int k, uint32_t* T_out, int* ties_out) {
  const int tid = threadIdx.x, rank = (int)cluster.block_rank();
  if (tid == 0) { sh.digit = 0; sh.remaining = k; }
  uint32_t prefix = 0;
  int remaining = k;
  const int shifts[3] = {21, 10, 0};
  const int widths[3] = {11, 11, 10};
  for (int p = 0; p < 3; ++p) {
    const int shift = shifts[p], width = widths[p];
    const uint32_t mask = (1u << width) - 1;
    for (int b = tid; b < kBins; b += kTopkThreads) sh.u.rx.hist[b] = 0;
    __syncthreads();
    // lanes that hit the same bin add once
    for (int64_t x0 = tid - (tid & 31); x0 < len; x0 += kTopkThreads) {
      const int64_t x = x0 + (tid & 31);
      const uint32_t key = x < len ? order_key(s[lo + x]) : 0u;
      const bool hit = x < len && (p == 0 || (key >> (shift + width)) == prefix);
      const uint32_t bin = hit ? (key >> shift) & mask : 0xFFFFFFFFu;
      if (!__any_sync(0xffffffffu, hit)) continue;
      const unsigned peers = __match_any_sync(0xffffffffu, bin);
      if (hit && (tid & 31) == __ffs(peers) - 1) atomicAdd(&sh.u.rx.hist[bin], __popc(peers));
    }
    // cluster reduce-scatter: CTA r sums bins [r*kBins/C, (r+1)*kBins/C)
    cluster.sync();
    constexpr int per = kBins / C;
    for (int b = tid; b < per; b += kTopkThreads) {
      int t = 0;
      for (int r = 0; r < C; ++r) t += cluster.map_shared_rank(&sh.u.rx.hist[0], r)[rank * per + b];
      sh.u.rx.slice_sum[b] = t;
    }
    cluster.sync();
    for (int b = tid; b < kBins; b += kTopkThreads)
      sh.u.rx.full[b] = cluster.map_shared_rank(&sh.u.rx.slice_sum[0], b / per)[b % per];
    __syncthreads();
    // digit d: the largest d with (count of digits > d) < remaining <= (count of digits >= d)
    {
      const int b0 = kBins - 2 - 2 * tid;        // 2 bins per thread, thread 0 owns the top bins
      const int c1 = sh.u.rx.full[b0 + 1], c0 = sh.u.rx.full[b0];
      int tot;
      const int before = block_excl_scan(c1 + c0, sh.wsum, &tot);
      if (before < remaining && before + c1 >= remaining) {
        sh.digit = (uint32_t)(b0 + 1);
        sh.remaining = remaining - before;
      } else if (before + c1 < remaining && before + c1 + c0 >= remaining) {
        sh.digit = (uint32_t)b0;
        sh.remaining = remaining - before - c1;
      }
      __syncthreads();
    }
    prefix = (prefix << width) | sh.digit;
    remaining = sh.remaining;
    cluster.sync();   // histograms are read remotely until every CTA has its copy
  }
  *T_out = prefix;
  *ties_out = remaining;
}

// Radix path output: each warp owns a contiguous sub-slice, walked 32 keys
// at a time, so that ballots give ordered positions.
template <int C>
__device__ void radix_output(cg::cluster_group& cluster, TopkShared& sh, const float* s, int64_t lo, int64_t len,
                             uint32_t T, int ties_needed, int32_t* out) {
  const int tid = threadIdx.x, rank = (int)cluster.block_rank();
  const int lane = tid & 31, wid = tid >> 5;
  const int64_t per_w = ((len + kWarps - 1) / kWarps + 31) / 32 * 32;
  const int64_t w_lo = (int64_t)wid * per_w < len ? (int64_t)wid * per_w : len;
  const int64_t w_hi = w_lo + per_w < len ? w_lo + per_w : len;
  const unsigned lt_mask = (1u << lane) - 1u;
  int gt = 0, eq = 0;
  for (int64_t x0 = w_lo; x0 < w_hi; x0 += 32) {
    const int64_t x = x0 + lane;
    const uint32_t key = x < w_hi ? order_key(s[lo + x]) : 0u;
    gt += __popc(__ballot_sync(0xffffffffu, x < w_hi && key > T));
    eq += __popc(__ballot_sync(0xffffffffu, x < w_hi && key == T));
  }
  int gt_tot, eq_tot;
  (void)block_excl_scan(lane == 0 ? gt : 0, sh.wsum, &gt_tot);
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
  int w_ties = take_cta - eq_before;
  w_ties = w_ties < 0 ? 0 : (w_ties > eq ? eq : w_ties);
  int tot_sel;
  const int w_pos0 = __shfl_sync(0xffffffffu, block_excl_scan(lane == 0 ? gt + w_ties : 0, sh.wsum, &tot_sel), 0);
  int pos = sel_before + w_pos0;
  int ties_seen = 0;
  for (int64_t x0 = w_lo; x0 < w_hi; x0 += 32) {
    const int64_t x = x0 + lane;
    const uint32_t key = x < w_hi ? order_key(s[lo + x]) : 0u;
    const bool is_eq = x < w_hi && key == T;
    const unsigned eqb = __ballot_sync(0xffffffffu, is_eq);
    const int tie_rank = ties_seen + __popc(eqb & lt_mask);
    const bool take = x < w_hi && (key > T || (is_eq && tie_rank < w_ties));
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) out[pos + __popc(tb & lt_mask)] = (int32_t)(lo + x);
    pos += __popc(tb);
    ties_seen += __popc(eqb);
  }
}

}  // namespace

template <int C>
__global__ void __cluster_dims__(C, 1, 1) __launch_bounds__(kTopkThreads, 1) topk_cluster_kernel(TopkArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  TopkShared& sh = *reinterpret_cast<TopkShared*>(smem_raw);
  uint32_t* keys = reinterpret_cast<uint32_t*>(smem_raw + (sizeof(TopkShared) + 127) / 128 * 128);
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = (int)cluster.block_rank();
  const int i = blockIdx.y;
  const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
  const float* s = a.scores + (int64_t)i * a.ld;
  int32_t* out = a.out + (int64_t)i * a.k;
  // Launched with programmatic serialization after the index kernel: the
  // scores and counts are read only once that grid has completed.  The next
  // kernel on the stream (the attention, launched the same way) may become
  // resident and start what does not depend on the indices; it waits for
  // this grid before reading them.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
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
  const int64_t chunk = ((N + C - 1) / C + 3) / 4 * 4;
  const int64_t lo = (int64_t)rank * chunk < N ? (int64_t)rank * chunk : N;
  const int64_t hi = lo + chunk < N ? lo + chunk : N;
  const int64_t len = hi - lo;

  // ---- 1. threshold from a sample (the same sample in every CTA)
  const int S = N < kSample ? (int)N : kSample;
  float sraw[kSamplePer];         // loads issued here, used after the bulk copy is on its way
  bool sok[kSamplePer];
  // 64 evenly spaced runs of 64 consecutive scores (coalesced loads); all of
  // them when N < 4096
#pragma unroll
  for (int e = 0; e < kSamplePer; ++e) {
    const int x = tid + e * kTopkThreads;
    sok[e] = x < S;
    const int64_t pos = S < kSample ? (int64_t)x : (int64_t)(x / 64) * (N / 64) + (x % 64);
    sraw[e] = sok[e] ? s[pos] : 0.f;
  }
  // ---- slice -> shared memory: one bulk copy of the 16-byte aligned part
  const bool cached = a.cache_keys != 0;
  const bool bulk = cached && ((reinterpret_cast<uintptr_t>(s + lo) & 15) == 0);
  const int64_t nbulk = bulk ? len / 4 * 4 : 0;
  if (cached && tid == 0) {
    tc::mbar_init(&sh.bar, 1);
    tc::fence_mbar_init();
    tc::mbar_arrive_expect_tx(&sh.bar, (uint32_t)(nbulk * 4));
    for (int64_t x = 0; x < nbulk; x += 8192) {
      const int64_t m = nbulk - x < 8192 ? nbulk - x : 8192;
      tc::bulk_g2s(keys + x, s + lo + x, (uint32_t)(m * 4), &sh.bar);
    }
  }
  if (cached)
    for (int64_t x = nbulk + tid; x < len; x += kTopkThreads) keys[x] = __float_as_uint(s[lo + x]);
  for (int b = tid; b < kBins; b += kTopkThreads) sh.sel_hist[b] = 0;   // block_select's invariant
  if (tid == 0) sh.n_list = 0;
  __syncthreads();   // the mbarrier is initialised before anyone waits on it

  uint32_t sv[kSamplePer];
#pragma unroll
  for (int e = 0; e < kSamplePer; ++e) sv[e] = sok[e] ? order_key(sraw[e]) : 0u;
  const float lam = (float)k * (float)S / (float)N;     // expected sampled keys above the k-th
  const int r = (int)ceilf(lam + 6.f * sqrtf(lam) + 8.f);
  uint32_t tau = 0;
  if (r <= S) {
    uint32_t smin, smax;
    int unused;
    block_minmax(sv, sok, sh.mm[0], &smin, &smax);
    tau = block_select(sv, sok, r, smin, smax, sh, &unused);
  }
  // all threads observe the copy's completion (bounded wait).  A CTA whose
  // copy did not arrive does not leave on its own: it reports a count of -1
  // in the count exchange below, and the whole cluster then leaves together
  // after one more cluster barrier, so that no CTA touches the shared memory
  // of a CTA that has gone.
  const bool arrived = !cached || __syncthreads_and(tc::mbar_wait(&sh.bar, 0)) != 0;

  // ---- 2. filter: count, exchange counts, write candidates to the leader
  // Each warp owns a contiguous sub-slice (a multiple of 128 keys when the
  // slice is in shared memory: each lane then reads 4 keys per 16-byte load).
  const int64_t per_w = cached ? ((len + kWarps - 1) / kWarps + 127) / 128 * 128
                               : ((len + kWarps - 1) / kWarps + 31) / 32 * 32;
  const int64_t w_lo = (int64_t)wid * per_w < len ? (int64_t)wid * per_w : len;
  const int64_t w_hi = w_lo + per_w < len ? w_lo + per_w : len;
  const uint4* k4 = reinterpret_cast<const uint4*>(keys);
  auto load4 = [&](int64_t x, uint32_t (&kv)[4], bool (&pass)[4]) {
    uint4 v = make_uint4(0, 0, 0, 0);
    if (x < w_hi) v = k4[x >> 2];
    const uint32_t raw[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      kv[e] = order_key(__uint_as_float(raw[e]));
      pass[e] = x + e < w_hi && kv[e] >= tau;
    }
  };
  int wc = 0;
  if (!arrived) {
    // nothing to count: the slice never reached shared memory
  } else if (cached) {
    int c = 0;
    for (int64_t x0 = w_lo; x0 < w_hi; x0 += 128) {
      uint32_t kv[4];
      bool pass[4];
      load4(x0 + 4 * lane, kv, pass);
      c += (int)pass[0] + (int)pass[1] + (int)pass[2] + (int)pass[3];
    }
    wc = __reduce_add_sync(0xffffffffu, c);
  } else {
    for (int64_t x0 = w_lo; x0 < w_hi; x0 += 8 * 32) {
      uint32_t kv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t x = x0 + u * 32 + lane;
        kv[u] = x < w_hi ? order_key(s[lo + x]) : 0u;
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int64_t x = x0 + u * 32 + lane;
        wc += __popc(__ballot_sync(0xffffffffu, x < w_hi && kv[u] >= tau));
      }
    }
  }
  int cta_cnt;
  const int w_before = __shfl_sync(0xffffffffu, block_scan1(lane == 0 ? wc : 0, sh.scan_a, &cta_cnt), 0);
  if (tid == 0) sh.n_cand = arrived ? cta_cnt : -1;
  cluster.sync();
  int base, total;
  bool abort_all;
  {   // lane q reads CTA q's count (all remote reads in flight at once)
    const int c = lane < C ? *cluster.map_shared_rank(&sh.n_cand, lane) : 0;
    base = __reduce_add_sync(0xffffffffu, lane < rank ? c : 0);
    total = __reduce_add_sync(0xffffffffu, c);
    abort_all = __any_sync(0xffffffffu, c < 0);   // the same decision in every CTA
  }
  if (abort_all) {
    if (!arrived && tid == 0 && a.err && atomicCAS(a.err, 0, (int32_t)kErrTimeout) == 0) a.err[1] = i;
    cluster.sync();   // every CTA has read every count before any leaves
    return;
  }
  const bool filter = total >= k && total <= kCandCap;   // the same in every CTA
  if (filter) {
    uint2* lc = cluster.map_shared_rank(&sh.u.cand[0], 0);
    int pos = base + w_before;
    const unsigned lt_mask = (1u << lane) - 1u;
    if (cached) {
      for (int64_t x0 = w_lo; x0 < w_hi; x0 += 128) {
        const int64_t x = x0 + 4 * lane;
        uint32_t kv[4];
        bool pass[4];
        load4(x, kv, pass);
        const int cnt = (int)pass[0] + (int)pass[1] + (int)pass[2] + (int)pass[3];
        int incl = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += y;
        }
        int p = pos + incl - cnt;
#pragma unroll
        for (int e = 0; e < 4; ++e)
          if (pass[e]) lc[p++] = make_uint2(kv[e], (uint32_t)(lo + x + e));
        pos += __shfl_sync(0xffffffffu, incl, 31);
      }
    } else {
      for (int64_t x0 = w_lo; x0 < w_hi; x0 += 8 * 32) {
        uint32_t kv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int64_t x = x0 + u * 32 + lane;
          kv[u] = x < w_hi ? order_key(s[lo + x]) : 0u;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int64_t x = x0 + u * 32 + lane;
          const bool pass = x < w_hi && kv[u] >= tau;
          const unsigned b = __ballot_sync(0xffffffffu, pass);
          if (pass) lc[pos + __popc(b & lt_mask)] = make_uint2(kv[u], (uint32_t)(lo + x));
          pos += __popc(b);
        }
      }
    }
    cluster.sync();   // the leader's list is complete; nobody reads another CTA after this
    if (rank != 0) return;

    // ---- 3. exact selection among the candidates (leader)
    const int M = total;
    uint32_t cv[kCandPer];
    bool cok[kCandPer];
    const int e0 = tid * kCandPer;                     // contiguous run, index order
#pragma unroll
    for (int e = 0; e < kCandPer; ++e) {
      cok[e] = e0 + e < M;
      cv[e] = cok[e] ? sh.u.cand[e0 + e].x : 0u;
    }
    uint32_t cmin, cmax;
    block_minmax(cv, cok, sh.mm[1], &cmin, &cmax);
    int ties_needed;
    const uint32_t T = block_select(cv, cok, k, tau, cmax, sh, &ties_needed);
    // one scan of (count > T, count == T) packed in 16-bit halves (counts <= kCandCap)
    int ngt = 0, neq = 0;
#pragma unroll
    for (int e = 0; e < kCandPer; ++e) {
      ngt += (cok[e] && cv[e] > T) ? 1 : 0;
      neq += (cok[e] && cv[e] == T) ? 1 : 0;
    }
    int packed_tot;
    const int packed = block_scan1(ngt | (neq << 16), sh.scan_b, &packed_tot);
    const int gt_before = packed & 0xFFFF, eq_before = packed >> 16;
    int seen = eq_before;
    unsigned take_bits = 0;
#pragma unroll
    for (int e = 0; e < kCandPer; ++e) {
      const bool is_eq = cok[e] && cv[e] == T;
      const bool t = cok[e] && (cv[e] > T || (is_eq && seen < ties_needed));
      seen += is_eq ? 1 : 0;
      if (t) take_bits |= 1u << e;
    }
    int p = gt_before + (eq_before < ties_needed ? eq_before : ties_needed);
#pragma unroll
    for (int e = 0; e < kCandPer; ++e)
      if (take_bits & (1u << e)) out[p++] = (int32_t)sh.u.cand[e0 + e].y;
    return;
  }

  // ---- radix path (every CTA of the cluster)
  uint32_t T;
  int ties_needed;
  radix_select<C>(cluster, sh, s, lo, len, k, &T, &ties_needed);
  radix_output<C>(cluster, sh, s, lo, len, T, ties_needed, out);
  cluster.sync();   // no CTA may leave while others still read its shared memory
}

size_t topk_smem_bytes(int64_t ld, int cluster, bool* cache) {
  const int64_t chunk = ((ld + cluster - 1) / cluster + 3) / 4 * 4;
  const size_t base = (sizeof(TopkShared) + 127) / 128 * 128;
  const size_t with = base + (size_t)chunk * 4;
  *cache = with <= 227 * 1024;
  return *cache ? with : base;
}

namespace {

template <int C>
cudaError_t launch_topk_c(const TopkArgs& a, size_t sm, cudaStream_t st) {
  cudaError_t e = cudaFuncSetAttribute(topk_cluster_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  if (C > 8) {
    e = cudaFuncSetAttribute(topk_cluster_kernel<C>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (e != cudaSuccess) return e;
  }
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(C, a.n);
  cfg.blockDim = dim3(kTopkThreads);
  cfg.dynamicSmemBytes = sm;
  cfg.stream = st;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, topk_cluster_kernel<C>, a);
  note_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// The occupancy answers below are cached per (device, size); calls may come
// from several host threads, so each cache is read and written under a lock.
std::mutex g_occupancy_mu;

// Whether this device can co-schedule a 16-CTA cluster of the kernel with
// `sm` bytes of shared memory (asked once per device and size).
bool cluster16_ok(size_t sm) {
  std::lock_guard<std::mutex> lock(g_occupancy_mu);
  static int cached_dev = -1;
  static size_t cached_sm = 0;
  static bool cached_ok = false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  if (dev == cached_dev && sm == cached_sm) return cached_ok;
  bool ok = false;
  if (cudaFuncSetAttribute(topk_cluster_kernel<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1) == cudaSuccess &&
      cudaFuncSetAttribute(topk_cluster_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) ==
          cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(16, 1, 1);
    cfg.blockDim = dim3(kTopkThreads, 1, 1);
    cfg.dynamicSmemBytes = sm;
    int nclusters = 0;
    ok = cudaOccupancyMaxActiveClusters(&nclusters, topk_cluster_kernel<16>, &cfg) == cudaSuccess && nclusters > 0;
  }
  cudaGetLastError();
  cached_dev = dev;
  cached_sm = sm;
  cached_ok = ok;
  return ok;
}

// How many clusters of C CTAs of the kernel, with `sm` bytes of shared
// memory each, the device holds at once (asked once per device, C and size).
template <int C>
int max_clusters(size_t sm) {
  std::lock_guard<std::mutex> lock(g_occupancy_mu);
  static int cached_dev = -1;
  static size_t cached_sm = 0;
  static int cached_n = 0;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (dev == cached_dev && sm == cached_sm) return cached_n;
  int n = 0;
  if (cudaFuncSetAttribute(topk_cluster_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm) ==
      cudaSuccess) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(C, 1, 1);
    cfg.blockDim = dim3(kTopkThreads, 1, 1);
    cfg.dynamicSmemBytes = sm;
    if (cudaOccupancyMaxActiveClusters(&n, topk_cluster_kernel<C>, &cfg) != cudaSuccess) n = 0;
  }
  cudaGetLastError();
  cached_dev = dev;
  cached_sm = sm;
  cached_n = n;
  return n;
}

}  // namespace

// Cluster size for n rows of ld scores on a GPU that should take them in
// one wave: the largest of 16, 8 and 4 whose n clusters are all resident at
// once (16 only where the device co-schedules it), else 4.
int topk_cluster_one_wave(int64_t ld, int n) {
  bool cache = false;
  const size_t sm16 = topk_smem_bytes(ld, 16, &cache);
  if (cluster16_ok(sm16) && n <= max_clusters<16>(sm16)) return 16;
  if (n <= max_clusters<8>(topk_smem_bytes(ld, 8, &cache))) return 8;
  return 4;
}

cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* n_valid, int n, int k,
                        int32_t* out, int32_t* err, int cluster, cudaStream_t st) {
  if (n > 65535) return cudaErrorInvalidValue;
  if (cluster == 16) {
    bool cache16 = false;
    const size_t sm16 = topk_smem_bytes(ld, 16, &cache16);
    if (!cluster16_ok(sm16)) cluster = 8;
  }
  bool cache = false;
  const size_t sm = topk_smem_bytes(ld, cluster, &cache);
  TopkArgs a{scores, ld, n_valid, n, k, out, err, cache ? 1 : 0};
  switch (cluster) {
    case 16: return launch_topk_c<16>(a, sm, st);
    case 8: return launch_topk_c<8>(a, sm, st);
    case 4: return launch_topk_c<4>(a, sm, st);
    case 1: return launch_topk_c<1>(a, sm, st);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace csa
