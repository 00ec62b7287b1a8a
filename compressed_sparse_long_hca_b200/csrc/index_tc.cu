// Lightning-indexer scores on the 5th-generation tensor cores
// (csa_index_scores).
//
// Page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力": the query's index
// heads are scored against every compressed index key after a ReLU; podcast
// summary page, section "2.1 推理与计算效率": the indexer path runs in FP4.
//   s_j = sum_h w_h * max(0, q^_h . k^_j),   q^, k^ MXFP4 (E2M1, E8M0 per 32)
//
// Shape of the work: per query an FP4 product [N keys x d_I] x [d_I x H_I]
// with N up to 262,144 and H_I = 64 whose A operand (the keys, 68 B each) is
// streamed once from HBM.  The cache stores the index keys of every 512-token
// page as one ready-made operand tile (codes in the no-swizzle K-major
// core-matrix order, scales in the 32 x 128-bit order of tcgen05.cp), so a
// 128-key tile is one bulk copy.  Two persistent CTAs per SM (their tcgen05
// issue latencies overlap) each own a contiguous range of tiles of the
// flattened (query, tile) list and run three roles:
//   * producer (warp 0): one bulk async copy per tile into a ring of
//     shared-memory stages;
//   * MMA (warp 1): one thread copies the tile's key scales into TMEM
//     (tcgen05.cp) and issues the block-scaled MMA
//     D[128 keys x 64 heads] = K^ Q^T (kind::mxf4, M=128, N=64, K=64 per
//     instruction) into one of four TMEM accumulators;
//   * epilogue (warps 2-9, two groups of four warps taking alternate tiles):
//     read a finished accumulator (one TMEM lane = one key, 64 columns = its
//     64 head dot products) and reduce sum_h w_h max(0, d_h) in a fixed
//     order.  At a query boundary they quantise the next query's index heads
//     to MXFP4 (the B operand and its scale chunk).
// Every key's score comes from the same instruction sequence whatever the
// grid, so launch variants and batch compositions return identical bits.
// All waits are bounded: a stuck pipeline records a timeout in the device
// error word, lets in-flight copies land, frees TMEM and returns.
#include "common.cuh"
#include "tc.cuh"

namespace csa {

namespace {

constexpr int kStagesPlain = 8;        // shared-memory stages of key tiles, csa_index_scores (two CTAs per SM)
constexpr int kStagesFused = 18;       // csa_index_topk (one CTA per SM: a tile's copy takes ~3 us to land,
                                       // so an SM needs ~150 KB in flight to stream at the HBM rate)
constexpr int kStagesMax = kStagesFused;
constexpr int kNAPlain = 3;            // TMEM accumulators (and key-scale buffers), csa_index_scores
constexpr int kNAFused = 6;            // csa_index_topk: one CTA per SM owns all 512 TMEM columns
constexpr int kNAMax = kNAFused;
constexpr int kEpiGroups = 2;          // epilogue groups, alternate tiles
constexpr int kGroupThreads = 128;     // one thread per key of a tile
constexpr int kEpiThreads = kEpiGroups * kGroupThreads;
constexpr int kThreads = 64 + kEpiThreads;   // warp 0 producer, warp 1 MMA, warps 2-9 epilogue
constexpr int kHeadsN = 64;            // MMA N (index heads, zero padded)
constexpr int kMaxCh = 4;              // d_I / 32 <= 4
constexpr int kTileBytes = kCsaPerPage * kMaxCh * 16 + kSfChunk;   // codes + scale chunk
constexpr int kPassTiles = 128;        // tiles per pass (page-table window in smem)
constexpr int kMaxSeg = 64;            // queries per pass
constexpr int kMaxQ = 256;             // queries whose tile counts are kept in shared memory
// TMEM columns: accumulator na at 64 na, the keys' scales of accumulator na
// at 64 NA + 4 na, the query's scales after them.  csa_index_scores: 256
// columns per CTA (two CTAs fill the SM's 512); csa_index_topk: 512.
template <int NA> struct TmemCols {
  static constexpr uint32_t alloc = NA * 64 + 4 * NA + 4 <= 256 ? 256 : 512;
  static constexpr uint32_t sfa = NA * 64;
  static constexpr uint32_t sfb = NA * 64 + 4 * NA;
};
static_assert(TmemCols<kNAPlain>::alloc == 256 && TmemCols<kNAFused>::alloc == 512, "TMEM budget");
// fused top-k (csa_index_topk)
constexpr int kHistBits = 12;          // histogram of the score keys' top 12 bits
constexpr int kHistBins = 1 << kHistBits;
constexpr int kHistShift = 32 - kHistBits;
constexpr int kCandCap = 8192;         // candidates the selecting CTA holds
constexpr uint64_t kWaitLimitNs = 1000000000ull;
constexpr int kScoreCache = 8192;      // scores of the CTA's own range kept in shared memory (fused top-k)
// The selection's candidates and its two bitmaps reuse the fused kernel's
// tile stages (free once the CTA's scoring is done).
constexpr int kBitmapWords = ((kStagesFused * kTileBytes - kCandCap * 8) / 8) & ~31;
constexpr int64_t kBitmapKeys = (int64_t)kBitmapWords * 32;   // keys each bitmap covers

// Dynamic shared memory: IdxSmem, then the tile stages (kTileBytes each),
// then (fused top-k) the score cache.  In the top-k phase the stages hold
// the selection's candidates (key, index) and its two bitmaps.
struct IdxSmem {
  uint8_t qb[kHeadsN * kMaxCh * 16];                 // query codes, core-matrix order
  uint8_t qsf[kSfChunk];                             // query scales, tcgen05.cp order
  alignas(16) float w[kHeadsN];
  int32_t pgs[kPassTiles];                           // pool page of every tile of the pass
  // segments of the pass: one per query touched
  int32_t seg_q[kMaxSeg];
  int32_t seg_n[kMaxSeg];
  int64_t seg_t0[kMaxSeg];
  int64_t seg_N[kMaxSeg];
  int32_t n_seg;
  int32_t q_tiles[kMaxQ];                            // tiles of query i (i < kMaxQ)
  int64_t q_N[kMaxQ];                                // keys of query i
  int64_t red[kThreads / 32];
  uint64_t full[kStagesMax], stage_empty[kStagesMax];
  uint64_t acc_full[kNAMax], acc_empty[kNAMax];
  uint64_t q_ready;
  uint64_t drain;
  uint32_t tmem_base;
  volatile int abort;
  // fused top-k
  uint32_t hist[kHistBins];                          // score-key histogram of the current segment
  int32_t wt[2][kThreads / 32];                      // warp totals of block scans (alternating)
  int32_t flw[kEpiThreads / 32];                     // epilogue warp totals (histogram flush)
  int32_t tk_q, tk_t0, tk_nt, tk_flag, tk_bin, tk_above, tk_M, tk_rem;
  int64_t tk_N, tk_before;
  uint32_t tk_digit;
};

constexpr size_t kSmemHead = (sizeof(IdxSmem) + 127) / 128 * 128;

__device__ __forceinline__ uint8_t* smem_tiles(IdxSmem& sm) { return reinterpret_cast<uint8_t*>(&sm) + kSmemHead; }
__device__ __forceinline__ uint2* smem_cand(IdxSmem& sm) { return reinterpret_cast<uint2*>(smem_tiles(sm)); }
__device__ __forceinline__ uint32_t* smem_bitmaps(IdxSmem& sm) {
  return reinterpret_cast<uint32_t*>(smem_tiles(sm) + (size_t)kCandCap * 8);
}

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
  // fused top-k only
  int k;
  int32_t* idx_out;       // [n][k]
  int32_t* hist_done;     // [n]  CTAs whose histogram of the query is flushed
  int32_t* cand_done;     // [n]  CTAs whose candidates of the query are written
  uint32_t* hist;         // [n][kHistBins]  the query's keys over their top 12 bits
  uint32_t* hist2;        // [n][2048]       candidates in the k-th bin over key bits 9 .. 19
  int32_t* qcount;        // [n]             candidates appended so far
  uint2* cand;            // [n][ld]         candidates (key, index), in no particular order
  int q_per_req;          // 0: decode queries; C > 0: chunk queries (visible_tokens)
};

// Number of 128-key tiles of query i (0 for an invalid query); N = its keys.
__device__ __forceinline__ int64_t query_tiles(const IndexTcArgs& a, int i, int64_t* n_keys, int* req_out) {
  const int req = a.req_ids[i];
  *req_out = req;
  if (req < 0 || req >= a.L.max_req) { *n_keys = 0; return 0; }
  const int64_t T = visible_tokens(a.L.lengths()[(int64_t)a.layer * a.L.max_req + req], a.q_per_req, i);
  const int64_t N = T > 0 ? T / kCsaM : 0;
  *n_keys = N;
  if (N > a.ld) return 0;
  return (N + kCsaPerPage - 1) / kCsaPerPage;
}

// Bounded wait that also gives up as soon as another role has aborted.
__device__ __forceinline__ bool wait_or_abort(IdxSmem& sm, uint64_t* bar, uint32_t parity) {
  if (tc::mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = tc::globaltimer_ns();
  for (uint32_t spin = 0;; ++spin) {
    if (tc::mbar_try_wait(bar, parity)) return true;
    if ((spin & 127u) == 127u) {
      if (sm.abort) return false;
      if (tc::globaltimer_ns() - t0 > 2000000000ull) { sm.abort = 1; return false; }
    }
  }
}


// ---------------------------------------------------------------- fused top-k
//
// Selection rule (as csa_topk): the k largest scores, equal scores to the
// lower index, -0.0 == +0.0, output ascending, -1 padding.  Scores become
// order-preserving 32-bit keys; the kernel's CTAs build a histogram of each
// query's keys over their top 12 bits while they score, wait (bounded) until
// every CTA of the query has flushed its part, find the bin b holding the
// k-th largest key, and write the keys of their own range with top bits >= b
// (the candidates) compactly, in index order, into the window of the
// candidate buffer that starts at their range's first key.  The last CTA to
// finish a query gathers the windows in order and selects exactly; when more
// than kCandCap keys fall in bins >= b (a huge tie class), it selects with a
// radix select over the query's whole score row instead.  Both are exact, so
// the indices equal csa_topk's.

__device__ __forceinline__ uint32_t score_key(float s) {
  const uint32_t b = __float_as_uint(s + 0.0f);       // -0.0 -> +0.0
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// CTA that owns flattened tile g when `total` tiles are split over G CTAs as
// [total * c / G, total * (c + 1) / G).
__device__ __forceinline__ int owner_cta(int64_t g, int64_t total, int G) {
  return (int)(((g + 1) * (int64_t)G - 1) / total);
}

__device__ __forceinline__ int ld_acquire(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Exclusive prefix sum over the CTA's threads in thread order; one barrier.
// `wt` must not be reused before another barrier.
__device__ __forceinline__ int cta_scan(int v, int32_t* wt, int* total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wt[w] = x;
  __syncthreads();
  const int tw = lane < kThreads / 32 ? wt[lane] : 0;
  *total = __reduce_add_sync(0xffffffffu, tw);
  return __reduce_add_sync(0xffffffffu, lane < w ? tw : 0) + x - v;
}

// Among `nbins` counts (thread t < 256 owns bins nbins-PER*(t+1) .. nbins-PER*t-1,
// highest first), find the bin d holding the r-th largest key: (count in bins
// > d) < r <= (count in bins >= d).  Publishes d in sm.tk_digit, the count
// above it in sm.tk_above and the count at or above it in sm.tk_M; returns
// false when fewer than r keys are counted.  Two barriers.
template <int PER>
__device__ bool find_bin(const uint32_t* bins, int r, IdxSmem& sm) {
  const int tid = threadIdx.x;
  int c[PER];
  int sum = 0;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const int b = 256 * PER - 1 - (PER * tid + e);     // descending
    c[e] = tid < 256 ? (int)bins[b] : 0;
    sum += c[e];
  }
  if (tid == 0) sm.tk_flag = 0;
  int tot;
  const int before = cta_scan(sum, sm.wt[0], &tot);
  if (tid < 256 && before < r && before + sum >= r) {
    int cum = before;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      if (cum < r && cum + c[e] >= r) {
        sm.tk_digit = (uint32_t)(256 * PER - 1 - (PER * tid + e));
        sm.tk_above = cum;
        sm.tk_M = cum + c[e];
        sm.tk_flag = 1;
      }
      cum += c[e];
    }
  }
  __syncthreads();
  return sm.tk_flag != 0;
}

// find_bin over the 256 PER counts of a global histogram: thread t < 256
// loads its PER bins (256 PER - PER(t+1) .. 256 PER - PER t - 1) with PER / 4
// vector loads, all in flight at once.
template <int PER>
__device__ bool find_bin_global(const uint32_t* gbins, int r, IdxSmem& sm) {
  const int tid = threadIdx.x;
  int c[PER];
  int sum = 0;
  if (tid < 256) {
    const uint4* src = reinterpret_cast<const uint4*>(gbins + 256 * PER - PER * (tid + 1));
    uint32_t v[PER];
#pragma unroll
    for (int x = 0; x < PER / 4; ++x) {
      const uint4 w = __ldcg(src + x);
      v[4 * x] = w.x; v[4 * x + 1] = w.y; v[4 * x + 2] = w.z; v[4 * x + 3] = w.w;
    }
#pragma unroll
    for (int e = 0; e < PER; ++e) { c[e] = (int)v[PER - 1 - e]; sum += c[e]; }   // descending bins
  } else {
#pragma unroll
    for (int e = 0; e < PER; ++e) c[e] = 0;
  }
  if (tid == 0) sm.tk_flag = 0;
  int tot;
  const int before = cta_scan(sum, sm.wt[0], &tot);
  if (tid < 256 && before < r && before + sum >= r) {
    int cum = before;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      if (cum < r && cum + c[e] >= r) {
        sm.tk_digit = (uint32_t)(256 * PER - 1 - (PER * tid + e));
        sm.tk_above = cum;
        sm.tk_M = cum + c[e];
        sm.tk_flag = 1;
      }
      cum += c[e];
    }
  }
  __syncthreads();
  return sm.tk_flag != 0;
}

// Histogram of the digit (key >> shift) & (2^bits - 1) over the keys whose
// higher bits (key >> (shift + bits)) equal `prefix`, into sm.hist[0 .. 2^bits);
// then find the bin of the r-th largest.  `keys(x)` yields key x of `count`.
template <int BITS, typename F>
__device__ bool digit_round(F keys, int64_t count, uint32_t prefix, int shift, int r, IdxSmem& sm) {
  for (int b = threadIdx.x; b < (1 << BITS); b += kThreads) sm.hist[b] = 0;
  __syncthreads();
  for (int64_t x = threadIdx.x; x < count; x += kThreads) {
    const uint32_t key = keys(x);
    if ((key >> (shift + BITS)) == prefix) atomicAdd(&sm.hist[(key >> shift) & ((1u << BITS) - 1)], 1u);
  }
  __syncthreads();
  return find_bin<(1 << BITS) / 256>(sm.hist, r, sm);
}

// The k-th largest key among `count` keys whose top 12 bits are >= `bin`,
// given `above` keys with top bits > bin: returns T and sets *ties = the
// number of keys == T that are selected.
template <typename F>
__device__ uint32_t exact_kth(F keys, int64_t count, uint32_t bin, int above, int k, IdxSmem& sm, int* ties,
                              bool* ok) {
  int r = k - above;
  *ok = digit_round<11>(keys, count, bin, 9, r, sm);           // bits 9 .. 19
  const uint32_t dA = sm.tk_digit;
  r -= sm.tk_above;
  const bool okB = digit_round<9>(keys, count, (bin << 11) | dA, 0, r, sm);   // bits 0 .. 8
  *ok = *ok && okB;
  const uint32_t dB = sm.tk_digit;
  *ties = r - sm.tk_above;
  __syncthreads();
  return (bin << 20) | (dA << 9) | dB;
}


// Add this CTA's histogram of query q's keys to the query's global histogram
// and clear it (epilogue thread et owns bins 16 et .. 16 et + 15; all
// epilogue threads call it).  Only the bins from the top down to the one
// holding this CTA's k-th largest key are added: the query's k-th largest key
// is at least as large as any CTA's k-th largest, so the global counts stay
// exact in every bin at or above the query's k-th bin, which is all the
// selection reads.
__device__ __forceinline__ void flush_hist(const IndexTcArgs& a, IdxSmem& sm, int q, int et) {
  constexpr int P = kHistBins / kEpiThreads;
  const int lane = et & 31, w = et >> 5;
  int mine = 0;
#pragma unroll
  for (int e = 0; e < P; ++e) mine += (int)sm.hist[et * P + e];
  // keys in the bins of the epilogue threads after this one (higher bins)
  int x = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_down_sync(0xffffffffu, x, o);
    if (lane + o < 32) x += y;
  }
  if (lane == 0) sm.flw[w] = x;
  tc::named_bar_sync(1, kEpiThreads);
  int above = x - mine;
  for (int v = w + 1; v < kEpiThreads / 32; ++v) above += sm.flw[v];
  uint32_t* g = a.hist + (int64_t)q * kHistBins;
#pragma unroll
  for (int e = P - 1; e >= 0; --e) {
    const uint32_t c = sm.hist[et * P + e];
    if (c) {
      if (above < a.k) atomicAdd(&g[et * P + e], c);
      sm.hist[et * P + e] = 0;
    }
    above += (int)c;
  }
  tc::named_bar_sync(1, kEpiThreads);                  // sm.flw may be reused
}

__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Inclusive prefix sum over the lanes of a warp.
__device__ __forceinline__ int warp_incl_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// A shared-memory bitmap of nw words read in chunks of 32 consecutive words
// (lane l of chunk c reads word 32 c + l, one word per bank), warp w owning
// chunks [c0, c1) in order.  Returns the number of set bits in the chunks of
// the warps before this one.  Two barriers; uses sm.wt[1].
__device__ __forceinline__ int bitmap_warp_base(const uint32_t* bm, int nw, int c0, int c1, IdxSmem& sm) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  int cnt = 0;
  for (int c = c0; c < c1; ++c) {
    const int x = c * 32 + lane;
    cnt += x < nw ? __popc(bm[x]) : 0;
  }
  cnt = __reduce_add_sync(0xffffffffu, cnt);
  if (lane == 0) sm.wt[1][w] = cnt;
  __syncthreads();
  const int tw = lane < kThreads / 32 ? sm.wt[1][lane] : 0;
  const int base = __reduce_add_sync(0xffffffffu, lane < w ? tw : 0);
  __syncthreads();
  return base;
}

// Write the selected indices of `count` keys (key(x), index(x) in index
// order): every key > T and the first `ties` keys == T, ascending.
template <typename FK, typename FI>
__device__ void write_selection(FK key, FI index, int64_t count, uint32_t T, int ties, int32_t* out, IdxSmem& sm,
                                const Layout& L, int req, int layer) {
  const int tid = threadIdx.x;
  const int64_t per = (count + kThreads - 1) / kThreads;
  const int64_t e0 = tid * per, e1 = e0 + per < count ? e0 + per : count;
  int ngt = 0, neq = 0;
  for (int64_t x = e0; x < e1; ++x) {
    const uint32_t v = key(x);
    ngt += v > T ? 1 : 0;
    neq += v == T ? 1 : 0;
  }
  int tot;
  const int gt_before = cta_scan(ngt, sm.wt[0], &tot);
  const int eq_before = cta_scan(neq, sm.wt[1], &tot);
  int p = gt_before + (eq_before < ties ? eq_before : ties);
  int seen = eq_before;
  for (int64_t x = e0; x < e1; ++x) {
    const uint32_t v = key(x);
    const bool eq = v == T;
    if (v > T || (eq && seen < ties)) out[p++] = index(x);
    seen += eq ? 1 : 0;
  }
  __syncthreads();
}

// The query's raw-token window ring into L2 (the attention's last rows).
__device__ __forceinline__ void prefetch_window(const Layout& L, int req, int layer) {
  const char* st = L.state(req, layer);
  for (int64_t o = threadIdx.x * 128; o < L.ring_bytes; o += (int64_t)kThreads * 128) prefetch_l2(st + o);
}

// The top-k part of csa_index_topk, by every thread of a CTA that scored the
// tiles [g0, g1) of the flattened (query, tile) list (its histograms flushed).
// The selection of query q by its last CTA (every CTA of q has flushed its
// histogram and appended its candidates): indices ascending into idx_out.
// bin / above / M: the k-th bin of the complete histogram, the keys above it
// and at or above it, as this CTA found them for its own filter.
__device__ void select_query(const IndexTcArgs& a, IdxSmem& sm, int q, int64_t N, uint32_t bin, int above, int M) {
  const Layout& L = a.L;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  __threadfence();
  int32_t* out = a.idx_out + (int64_t)q * a.k;
  const int req = a.req_ids[q];
  const float* row = a.scores + (int64_t)q * a.ld;
  const uint2* cq = a.cand + (int64_t)q * a.ld;
  prefetch_window(L, req, a.layer);
  if (N <= a.k) {                               // every entry is selected
    for (int j = tid; j < a.k; j += kThreads) out[j] = j < N ? j : -1;
    __syncthreads();
    return;
  }
    if (M <= kCandCap && N <= kBitmapKeys) {
      // first digit of the k-th key (bits 9 .. 19) from the candidates' hist2
      const int r1 = a.k - above;
      bool ok = find_bin_global<8>(a.hist2 + (int64_t)q * 2048, r1, sm);
      const uint32_t dA = sm.tk_digit;
      const int r2 = r1 - sm.tk_above;
      const int Mtot = __ldcg(a.qcount + q);
      __syncthreads();
      if (!ok || Mtot != M) {                   // cannot happen unless a CTA skipped its part
        if (tid == 0) {
          int32_t* e = L.err();
          if (atomicCAS(e, 0, (int32_t)kErrBounds) == 0) {
            e[1] = 7000000 + q;
            e[2] = M;
            e[3] = Mtot | (ok ? 0 : (1 << 30));
          }
        }
        return;
      }
      // the candidates to shared memory (no order needed), all loads in flight
      uint2* cand = smem_cand(sm);
      constexpr int kB = 8;
      for (int m0 = 0; m0 < Mtot; m0 += kThreads * kB) {
        uint2 v[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const int m = m0 + u * kThreads + tid;
          v[u] = m < Mtot ? __ldcg(cq + m) : make_uint2(0, 0);
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const int m = m0 + u * kThreads + tid;
          if (m < Mtot) cand[m] = v[u];
        }
      }
      __syncthreads();
      // last digit (bits 0 .. 8) among the candidates that share T's upper 23 bits
      const uint32_t pre = (bin << 11) | dA;
      ok = digit_round<9>([&](int64_t x) { return cand[x].x; }, Mtot, pre, 0, r2, sm);
      const uint32_t T = (pre << 9) | sm.tk_digit;
      const int ties = r2 - sm.tk_above;        // keys == T to take, lowest indices first
      const int n_eq = sm.tk_M - sm.tk_above;   // keys == T among the candidates
      __syncthreads();
      if (!ok) {
        if (tid == 0) set_err(L, kErrBounds, 7100000 + q);
        return;
      }
      // bitmaps over the query's N keys: selected and (when only some of the
      // keys == T are taken) the tied ones
      uint32_t* mb = smem_bitmaps(sm);
      uint32_t* tb = mb + kBitmapWords;
      const int nw = (int)((N + 31) / 32);
      const bool all_ties = ties == n_eq;       // the usual case: every key == T is taken
      for (int x = tid; x < nw; x += kThreads) {
        mb[x] = 0;
        if (!all_ties) tb[x] = 0;
      }
      __syncthreads();
      for (int m = tid; m < Mtot; m += kThreads) {
        const uint2 c = cand[m];
        if (c.x > T || (all_ties && c.x == T)) atomicOr(mb + (c.y >> 5), 1u << (c.y & 31));
        else if (c.x == T) atomicOr(tb + (c.y >> 5), 1u << (c.y & 31));
      }
      __syncthreads();
      const int nc = (nw + 31) / 32;            // chunks of 32 words, lane l reads word 32 c + l
      const int cpw = (nc + kThreads / 32 - 1) / (kThreads / 32);
      const int c0 = min(warp * cpw, nc), c1 = min(c0 + cpw, nc);
      if (!all_ties) {
        // the `ties` lowest tied indices join the selection
        int base = bitmap_warp_base(tb, nw, c0, c1, sm);
        for (int c = c0; c < c1; ++c) {
          const int x = c * 32 + lane;
          uint32_t t = x < nw ? tb[x] : 0u;
          const int n = __popc(t);
          const int incl = warp_incl_scan(n, lane);
          const int before = base + incl - n;
          if (before >= ties) {
            t = 0;
          } else if (before + n > ties) {       // keep the lowest (ties - before) bits
            uint32_t keep = 0;
            for (int j = ties - before; j > 0; --j) {
              keep |= t & (0u - t);
              t &= t - 1;
            }
            t = keep;
          }
          if (x < nw) mb[x] |= t;
          base += __shfl_sync(0xffffffffu, incl, 31);
        }
        __syncthreads();
      }
      // every selected index, ascending: staged in shared memory (the
      // candidates are no longer needed), then written out coalesced
      int32_t* staged = reinterpret_cast<int32_t*>(cand);
      int p = bitmap_warp_base(mb, nw, c0, c1, sm);
      for (int c = c0; c < c1; ++c) {
        const int x = c * 32 + lane;
        uint32_t b = x < nw ? mb[x] : 0u;
        const int n = __popc(b);
        const int incl = warp_incl_scan(n, lane);
        int o = p + incl - n;
        while (b) {
          staged[o++] = x * 32 + (__ffs(b) - 1);
          b &= b - 1;
        }
        p += __shfl_sync(0xffffffffu, incl, 31);
      }
      __syncthreads();
      for (int x = tid; x < a.k; x += kThreads) out[x] = staged[x];
      __syncthreads();
    } else {
      // more keys than kCandCap at or above the bin (a huge tie class):
      // radix select over the whole score row
      int ties;
      bool ok;
      auto rk = [&](int64_t x) { return score_key(__ldcg(row + x)); };
      const uint32_t T = exact_kth(rk, N, bin, above, a.k, sm, &ties, &ok);
      if (!ok) {
        if (tid == 0) set_err(L, kErrBounds, 7200000 + q);
        return;
      }
      write_selection(rk, [&](int64_t x) { return (int32_t)x; }, N, T, ties, out, sm, L, req, a.layer);
    }
}

__device__ void topk_phase(const IndexTcArgs& a, IdxSmem& sm, int64_t total, int64_t g0, int64_t g1,
                           const float* sc_cache) {
  const Layout& L = a.L;
  const int tid = threadIdx.x, lane = tid & 31;
  const int G = gridDim.x;
  tc::griddep_launch_dependents();    // the next kernel may start launching while the selection runs
  __threadfence();
  __syncthreads();
  // thread 0 walks the queries whose tiles overlap [g0, g1)
  int walk_q = 0;
  int64_t walk_before = 0;
  auto next_covered = [&](int& q, int64_t& before, int& nt, int64_t& N) {
    q = -1;
    while (walk_q < a.n && walk_before < g1) {
      int64_t n_keys;
      int req;
      const int64_t t = walk_q < kMaxQ ? sm.q_tiles[walk_q] : query_tiles(a, walk_q, &n_keys, &req);
      if (walk_q < kMaxQ) n_keys = sm.q_N[walk_q];
      const int64_t b0 = walk_before;
      walk_before += t;
      const int qq = walk_q++;
      if (t > 0 && b0 + t > g0) {
        q = qq; before = b0; nt = (int)t; N = n_keys;
        return;
      }
    }
  };
  // 1. arrive on every covered query's histogram counter
  if (tid == 0) {
    int q, nt;
    int64_t before, N;
    for (next_covered(q, before, nt, N); q >= 0; next_covered(q, before, nt, N)) atomicAdd(&a.hist_done[q], 1);
    walk_q = 0;
    walk_before = 0;
  }
  // 2. per covered query: threshold, candidates, and the selection by the last CTA
  for (;;) {
    if (tid == 0) {
      int q, nt;
      int64_t before, N;
      next_covered(q, before, nt, N);
      sm.tk_q = q;
      sm.tk_before = before;
      sm.tk_nt = nt;
      sm.tk_N = N;
    }
    __syncthreads();
    const int q = sm.tk_q;
    if (q < 0) break;
    const int64_t before = sm.tk_before, N = sm.tk_N;
    const int nt_q = sm.tk_nt;
    // the CTAs holding tiles of q: owners of its first and last tile and every
    // non-empty CTA between them (a CTA whose share rounds to no tile takes no part)
    const int c_first = owner_cta(before, total, G), c_last = owner_cta(before + nt_q - 1, total, G);
    int n_ctas;
    {
      const int c = c_first + tid;
      const int64_t gs = total * c / G, ge = total * (c + 1) / G;
      const bool holds = c <= c_last && gs < ge;
      (void)cta_scan(holds ? 1 : 0, sm.wt[0], &n_ctas);
      __syncthreads();
    }
    const int64_t lo_t = (g0 > before ? g0 : before) - before;
    const int64_t hi_t = (g1 < before + nt_q ? g1 : before + nt_q) - before;
    const bool all = N <= a.k;                 // every entry is selected
    const float* row = a.scores + (int64_t)q * a.ld;
    uint2* cq = a.cand + (int64_t)q * a.ld;
    bool fine = true;
    uint32_t bin = 0;
    int above = 0, M = 0;
    if (!all) {
      if (tid == 0) {
        bool ok = ld_acquire(&a.hist_done[q]) >= n_ctas;
        if (!ok) {
          const uint64_t t0 = tc::globaltimer_ns();
          while (!(ok = ld_acquire(&a.hist_done[q]) >= n_ctas) && tc::globaltimer_ns() - t0 < kWaitLimitNs)
            __nanosleep(100);
        }
        if (!ok) set_err(L, kErrTimeout, 6000000 + q);
        sm.tk_flag = ok ? 1 : 0;
      }
      __syncthreads();
      fine = sm.tk_flag != 0;
      __syncthreads();
      if (fine) {
        fine = find_bin_global<kHistBins / 256>(a.hist + (int64_t)q * kHistBins, a.k, sm);
        bin = sm.tk_digit;
        above = sm.tk_above;
        M = sm.tk_M;
        __syncthreads();
      }
      if (fine && M <= kCandCap) {
        // this CTA's keys of q with top bits >= bin (the candidates) are
        // appended to the query's candidate array, in no particular order:
        // a first pass counts them per warp, one global atomic reserves the
        // CTA's range, a second pass writes them.  Those in the k-th bin are
        // also counted over key bits 9 .. 19 for the selection's first digit.
        const int64_t j_lo = lo_t * kCsaPerPage, j_hi = hi_t * kCsaPerPage < N ? hi_t * kCsaPerPage : N;
        const int warp = tid >> 5;
        const unsigned lt = (1u << lane) - 1u;
        constexpr int kB = 8;                   // keys per lane in flight
        // the CTA's own scores of q: in the shared-memory cache (local index of
        // key j = (first local tile of q) * 128 + j - j_lo) or, past it, in L2
        const float* cache = sc_cache != nullptr ? sc_cache + ((before + lo_t - g0) * kCsaPerPage - j_lo) : nullptr;
        uint32_t* h2 = a.hist2 + (int64_t)q * 2048;
        auto load = [&](int64_t base, float (&v)[kB]) {
#pragma unroll
          for (int u = 0; u < kB; ++u) {
            const int64_t j = base + u * 32 + lane;
            v[u] = j < j_hi ? (cache != nullptr ? cache[j] : __ldcg(row + j)) : 0.f;
          }
        };
        const int64_t stride = (int64_t)(kThreads / 32) * 32 * kB;
        int cnt = 0;
        for (int64_t base = j_lo + (int64_t)warp * 32 * kB; base < j_hi; base += stride) {
          float v[kB];
          load(base, v);
#pragma unroll
          for (int u = 0; u < kB; ++u) {
            const int64_t j = base + u * 32 + lane;
            cnt += __popc(__ballot_sync(0xffffffffu, j < j_hi && (score_key(v[u]) >> kHistShift) >= bin));
          }
        }
        // warp totals -> the warp's offset in the CTA's range, one atomic per CTA
        int tot_c;
        const int wbase = cta_scan(lane == 0 ? cnt : 0, sm.wt[1], &tot_c);
        if (tid == 0) sm.tk_rem = tot_c > 0 ? atomicAdd(a.qcount + q, tot_c) : 0;
        __syncthreads();
        int off = sm.tk_rem + __shfl_sync(0xffffffffu, wbase, 0);
        for (int64_t base = j_lo + (int64_t)warp * 32 * kB; base < j_hi; base += stride) {
          float v[kB];
          load(base, v);
#pragma unroll
          for (int u = 0; u < kB; ++u) {
            const int64_t j = base + u * 32 + lane;
            const uint32_t key = score_key(v[u]);
            const bool pass = j < j_hi && (key >> kHistShift) >= bin;
            const unsigned bal = __ballot_sync(0xffffffffu, pass);
            if (pass) {
              cq[off + __popc(bal & lt)] = make_uint2(key, (uint32_t)j);
              if ((key >> kHistShift) == bin) atomicAdd(h2 + ((key >> 9) & 2047u), 1u);
            }
            off += __popc(bal);
          }
        }
      }
    }
    // arrive; the last CTA of the query selects (its candidates and bitmaps
    // go to the tile stages, apart from the score cache later filters read)
    __threadfence();
    __syncthreads();
    if (tid == 0) sm.tk_flag = atomicAdd(&a.cand_done[q], 1) == n_ctas - 1 ? 1 : 0;
    __syncthreads();
    const bool last = sm.tk_flag != 0;
    __syncthreads();
    if (last) {
      if (all || fine) select_query(a, sm, q, N, bin, above, M);
      else if (tid == 0) set_err(L, kErrBounds, 7300000 + q);   // the bin was never found
    }
  }
}

}  // namespace

template <bool kTopk>
__global__ void __launch_bounds__(kThreads, kTopk ? 1 : 2) index_tc_kernel(IndexTcArgs a) {
  constexpr int kStages = kTopk ? kStagesFused : kStagesPlain;
  constexpr int kNA = kTopk ? kNAFused : kNAPlain;
  constexpr uint32_t kTmemCols = TmemCols<kNA>::alloc, kSfaCol = TmemCols<kNA>::sfa, kSfbCol = TmemCols<kNA>::sfb;
  extern __shared__ __align__(128) uint8_t smem_raw[];
  IdxSmem& sm = *reinterpret_cast<IdxSmem*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  uint8_t* const tiles = smem_tiles(sm);
  const Layout& L = a.L;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int HI = L.HI, dI = L.dI, CH = dI / 32, CHs = L.CHs;
  const int n_mma = CHs / 2;                        // K = 64 per instruction
  const uint32_t sbo = (uint32_t)CHs * 128;
  const uint32_t tile_bytes = (uint32_t)L.idx_tile_bytes;
  const uint32_t sf_off = (uint32_t)(kCsaPerPage * CHs * 16);

  // ---- set-up (overlaps the bookkeeping's global loads below)
  if (warp == 1) {
    tc::tmem_alloc(&sm.tmem_base, kTmemCols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) { tc::mbar_init(&sm.full[s], 1); tc::mbar_init(&sm.stage_empty[s], 1); }
    for (int k = 0; k < kNA; ++k) { tc::mbar_init(&sm.acc_full[k], 1); tc::mbar_init(&sm.acc_empty[k], kGroupThreads); }
    tc::mbar_init(&sm.q_ready, 1);
    tc::mbar_init(&sm.drain, 1);
    sm.abort = 0;
    tc::fence_mbar_init();
  }

  // ---- per-query bookkeeping (one thread per query); every CTA computes
  //      the same tile total
  int64_t total = 0;
  {
    int64_t part = 0;
    for (int i = tid; i < a.n; i += kThreads) {
      int64_t N;
      int req;
      const int64_t nt = query_tiles(a, i, &N, &req);
      if (i < kMaxQ) { sm.q_tiles[i] = (int32_t)nt; sm.q_N[i] = N; }
      part += nt;
      if (blockIdx.x == 0) {
        // a query without tiles takes no part in the fused selection: its row is all -1
        if (kTopk && nt == 0)
          for (int j = 0; j < a.k; ++j) a.idx_out[(int64_t)i * a.k + j] = -1;
        if (req < 0 || req >= L.max_req) { set_err(L, kErrBounds, i); a.n_valid[i] = 0; continue; }
        a.n_valid[i] = (int32_t)N;
        if (N > a.ld) set_err(L, kErrLd, i);
      }
    }
    if (kTopk)
      for (int b = tid; b < kHistBins; b += kThreads) sm.hist[b] = 0;
    for (int o = 16; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
    if (lane == 0) sm.red[warp] = part;
    tc::tc_fence_before();
    __syncthreads();                       // also publishes the TMEM address and the barriers
    tc::tc_fence_after();
    for (int w = 0; w < kThreads / 32; ++w) total += sm.red[w];
  }
  const uint32_t tmem = sm.tmem_base;
  const int64_t g0 = total * blockIdx.x / gridDim.x, g1 = total * (blockIdx.x + 1) / gridDim.x;
  // fused top-k: the scores of this CTA's range also go to shared memory when they fit
  float* sc_cache = (kTopk && (g1 - g0) * kCsaPerPage <= kScoreCache)
                        ? reinterpret_cast<float*>(tiles + (size_t)kStages * kTileBytes)
                        : nullptr;
  if (g0 >= g1) {                          // no tiles for this CTA: nothing was issued
    if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);
    return;
  }

  // role state (each role only uses its own)
  int hist_q = -1;           // epilogue, fused top-k: query whose keys sm.hist counts
  uint32_t u_base = 0;       // CTA-wide tile counter at the start of the pass (barrier phases)
  uint32_t seg_count = 0;    // segments processed (q_ready phases)
  uint32_t n_issued = 0;     // producer: tiles whose copy has been issued (tiles 0 .. n_issued-1)
  int qi = 0;
  int64_t before = 0;        // tiles of queries < qi
  int64_t g = g0;

  while (g < g1 && !sm.abort) {
    // ---- pass prologue: segment table and page window (all threads)
    __syncthreads();
    if (tid == 0) {
      int ns = 0;
      int64_t gg = g, used = 0;
      while (gg < g1 && used < kPassTiles && ns < kMaxSeg) {
        int64_t N, nt;
        if (qi < kMaxQ) {
          nt = sm.q_tiles[qi];
          N = sm.q_N[qi];
        } else {
          int req;
          nt = query_tiles(a, qi, &N, &req);
        }
        if (nt == 0 || before + nt <= gg) { before += nt; ++qi; continue; }
        const int64_t t0 = gg - before;
        int64_t cnt = (g1 - before < nt ? g1 - before : nt) - t0;
        if (cnt > kPassTiles - used) cnt = kPassTiles - used;
        sm.seg_q[ns] = qi;
        sm.seg_t0[ns] = t0;
        sm.seg_n[ns] = (int32_t)cnt;
        sm.seg_N[ns] = N;
        ++ns;
        used += cnt;
        gg += cnt;
      }
      sm.n_seg = ns;
    }
    __syncthreads();
    {
      int base = 0;
      for (int sg = 0; sg < sm.n_seg; ++sg) {
        const int32_t* pt = L.page_table(a.req_ids[sm.seg_q[sg]]);
        for (int x = tid; x < sm.seg_n[sg]; x += kThreads) sm.pgs[base + x] = pt[sm.seg_t0[sg] + x];
        base += sm.seg_n[sg];
      }
    }
    __syncthreads();
    const int n_seg = sm.n_seg;
    int pass_tiles = 0;
    for (int sg = 0; sg < n_seg; ++sg) pass_tiles += sm.seg_n[sg];

    if (warp == 0) {
      // ================= producer: one bulk copy per tile =================
      // The whole warp walks the loop; one elected lane issues.
      for (int k = 0; k < pass_tiles; ++k) {
        const uint32_t u = u_base + (uint32_t)k;
        const int s = u % kStages;
        const bool ok = u < (uint32_t)kStages || wait_or_abort(sm, &sm.stage_empty[s], ((u / kStages) - 1) & 1);
        if (!__all_sync(0xffffffffu, ok)) break;
        const char* src = L.page(sm.pgs[k], a.layer) + L.pg_idx_codes;
        if (tc::elect_one()) {
          tc::mbar_arrive_expect_tx(&sm.full[s], tile_bytes);
          tc::bulk_g2s(tiles + (size_t)s * kTileBytes, src, tile_bytes, &sm.full[s]);
        }
        __syncwarp();
        n_issued = u + 1;
      }
    } else if (warp == 1) {
      // ================= MMA issuer =================
      // The whole warp walks the loop; one elected lane issues the tcgen05
      // operations, whose operands are warp-uniform.
      uint32_t u = u_base;
      bool ok = true;
      for (int sg = 0; sg < n_seg && ok; ++sg) {
        ok = wait_or_abort(sm, &sm.q_ready, seg_count & 1);
        ++seg_count;
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc::tc_fence_after();
        if (tc::elect_one()) tc::tmem_cp_32x128b_x4(tmem + kSfbCol, tc::smem_desc(tc::smem_u32(sm.qsf), 128, 128));
        __syncwarp();
        const int nt = sm.seg_n[sg];
        for (int k = 0; k < nt; ++k, ++u) {
          const int s = u % kStages, na = u % kNA;
          ok = wait_or_abort(sm, &sm.full[s], (u / kStages) & 1) &&
               (u < (uint32_t)kNA || wait_or_abort(sm, &sm.acc_empty[na], ((u / kNA) - 1) & 1));
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc::tc_fence_after();
          const uint32_t a_base = tc::smem_u32(tiles + (size_t)s * kTileBytes);
          const uint32_t b_base = tc::smem_u32(sm.qb);
          const uint32_t sfa_col = tmem + kSfaCol + 4 * na;
          if (tc::elect_one()) {
            tc::tmem_cp_32x128b_x4(sfa_col, tc::smem_desc(a_base + sf_off, 128, 128));
            for (int m = 0; m < n_mma; ++m) {
              const uint64_t ad = tc::smem_desc(a_base + m * 256, 128, sbo);
              const uint64_t bd = tc::smem_desc(b_base + m * 256, 128, sbo);
              const uint32_t id = tc::idesc_mxf4(128, kHeadsN, 2 * m, 2 * m);
              tc::mma_mxf4(tmem + 64 * na, ad, bd, id, sfa_col | ((uint32_t)(2 * m) << 30),
                           (tmem + kSfbCol) | ((uint32_t)(2 * m) << 30), m > 0 ? 1u : 0u);
            }
            tc::mma_commit(&sm.acc_full[na]);
            tc::mma_commit(&sm.stage_empty[s]);
          }
          __syncwarp();
        }
      }
    } else {
      // ================= epilogue warps =================
      const int et = tid - 64;                       // 0 .. kEpiThreads-1
      const int grp = et / kGroupThreads;            // this group takes tiles u with u % kEpiGroups == grp
      const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
      const int key_in_tile = (warp & 3) * 32 + lane;
      uint32_t u = u_base;
      bool ok = true;
      // Every epilogue thread walks all segments and reaches every named
      // barrier, also after an abort (the work is then skipped), so that no
      // thread can be left waiting at a barrier another thread has left.
      for (int sg = 0; sg < n_seg; ++sg) {
        const int qq = sm.seg_q[sg];
        const int nt = sm.seg_n[sg];
        const int64_t t0 = sm.seg_t0[sg], N = sm.seg_N[sg];
        // -- all tiles of earlier segments are finished: every MMA that read
        //    the previous query's operands has completed.  Quantise this
        //    query's index heads: B operand codes and its scale chunk.
        tc::named_bar_sync(1, kEpiThreads);
        if (kTopk && hist_q != qq) {             // a new query: hand the last one's counts on
          if (hist_q >= 0) flush_hist(a, sm, hist_q, et);
          hist_q = qq;
        }
        for (int x = et; x < kHeadsN * CHs; x += kEpiThreads)
          reinterpret_cast<uint4*>(sm.qb)[x] = make_uint4(0, 0, 0, 0);
        for (int x = et; x < kSfChunk / 4; x += kEpiThreads)
          reinterpret_cast<uint32_t*>(sm.qsf)[x] = 0x7F7F7F7Fu;        // scale 1.0 for padding
        tc::named_bar_sync(1, kEpiThreads);
        const float* q = a.q_idx + (int64_t)qq * HI * dI;
        for (int blk = et; blk < HI * CH; blk += kEpiThreads) {
          const int h = blk / CH, c = blk % CH;
          const float4* src = reinterpret_cast<const float4*>(q + h * dI + c * 32);
          float v[32];
#pragma unroll
          for (int x = 0; x < 8; ++x) {
            const float4 f = src[x];
            v[4 * x] = f.x; v[4 * x + 1] = f.y; v[4 * x + 2] = f.z; v[4 * x + 3] = f.w;
          }
          float am = 0.f;
#pragma unroll
          for (int x = 0; x < 32; ++x) am = fmaxf(am, fabsf(v[x]));
          const int e = mx_exponent(am);
          uint32_t pk[4] = {0, 0, 0, 0};
#pragma unroll
          for (int x = 0; x < 16; ++x)
            pk[x >> 2] |= (uint32_t)e2m1x2_rn(scale_pow2(v[2 * x], e), scale_pow2(v[2 * x + 1], e)) << (8 * (x & 3));
          *reinterpret_cast<uint4*>(&sm.qb[(h >> 3) * sbo + c * 128 + (h & 7) * 16]) =
              make_uint4(pk[0], pk[1], pk[2], pk[3]);
          sm.qsf[Layout::idx_sf_off(h, c)] = (uint8_t)(e + 127);
        }
        for (int h = et; h < kHeadsN; h += kEpiThreads) sm.w[h] = h < HI ? a.w[(int64_t)qq * HI + h] : 0.f;
        tc::fence_proxy_async_smem();
        tc::named_bar_sync(1, kEpiThreads);
        if (et == 0) tc::mbar_arrive(&sm.q_ready);
        float* out = a.scores + (int64_t)qq * a.ld;
        for (int k = (int)((grp + kEpiGroups - (int)(u % kEpiGroups)) % kEpiGroups); k < nt && ok;
             k += kEpiGroups) {
          const uint32_t uk = u + (uint32_t)k;
          const int na = uk % kNA;
          if (!(ok = wait_or_abort(sm, &sm.acc_full[na], (uk / kNA) & 1))) break;
          tc::tc_fence_after();
          // four quarters of 16 head columns (few live registers); four
          // interleaved partial sums (heads h = 4i + p), combined in a fixed order
          const uint32_t col = tmem + lane_base + 64 * na;
          const float4* w4 = reinterpret_cast<const float4*>(sm.w);
          float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;
          auto accumulate = [&](int qtr, const uint32_t* r) {
#pragma unroll
            for (int h4 = 0; h4 < 4; ++h4) {
              if (16 * qtr + h4 * 4 < HI) {
                const float4 wv = w4[4 * qtr + h4];
                p0 = fmaf(wv.x, fmaxf(__uint_as_float(r[4 * h4 + 0]), 0.f), p0);
                p1 = fmaf(wv.y, fmaxf(__uint_as_float(r[4 * h4 + 1]), 0.f), p1);
                p2 = fmaf(wv.z, fmaxf(__uint_as_float(r[4 * h4 + 2]), 0.f), p2);
                p3 = fmaf(wv.w, fmaxf(__uint_as_float(r[4 * h4 + 3]), 0.f), p3);
              }
            }
          };
          if constexpr (kTopk) {
            // registers to spare (one CTA per SM): all four loads, one wait
            uint32_t r[4][16];
#pragma unroll
            for (int qtr = 0; qtr < 4; ++qtr) tc::tmem_ld_x16(col + 16 * qtr, r[qtr]);
            tc::tmem_wait_ld();
            tc::tc_fence_before();
            tc::mbar_arrive(&sm.acc_empty[na]);
#pragma unroll
            for (int qtr = 0; qtr < 4; ++qtr) accumulate(qtr, r[qtr]);
          } else {
#pragma unroll
            for (int qtr = 0; qtr < 4; ++qtr) {
              uint32_t r[16];
              tc::tmem_ld_x16(col + 16 * qtr, r);
              tc::tmem_wait_ld();
              if (qtr == 3) {
                tc::tc_fence_before();
                tc::mbar_arrive(&sm.acc_empty[na]);
              }
              accumulate(qtr, r);
            }
          }
          const int64_t j = (t0 + k) * kCsaPerPage + key_in_tile;
          if (j < N) {
            const float sc = (p0 + p1) + (p2 + p3);
            out[j] = sc;
            if (kTopk) {
              atomicAdd(&sm.hist[score_key(sc) >> kHistShift], 1u);
              if (sc_cache != nullptr) sc_cache[(int64_t)uk * kCsaPerPage + key_in_tile] = sc;
            }
          }
        }
        u += (uint32_t)nt;
        if (!ok) sm.abort = 1;
      }
    }
    u_base += (uint32_t)pass_tiles;
    g += pass_tiles;
    __syncthreads();
  }
  // csa_index_scores: the next kernel on the stream (the top-k, launched with
  // programmatic serialization) may start launching; it waits for this grid
  // before reading the scores
  if (!kTopk) tc::griddep_launch_dependents();
  if (warp == 1 && u_base > 0) {
    // every tcgen05 operation this CTA issued has finished before TMEM is released
    if (tc::elect_one()) tc::mma_commit(&sm.drain);
    __syncwarp();
    tc::mbar_wait(&sm.drain, 0, 200000000ull);
  }
  if (sm.abort) {
    if (tid == 0) {
      set_err(L, kErrTimeout, blockIdx.x);
      // let copies already in flight land before the shared memory goes away
      for (int s = 0; s < kStages && (uint32_t)s < n_issued; ++s) {
        const uint32_t last = (uint32_t)s + kStages * ((n_issued - 1 - (uint32_t)s) / kStages);   // last tile of stage s
        tc::mbar_wait(&sm.full[s], (last / kStages) & 1, 200000000ull);
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) tc::tmem_dealloc(tmem, kTmemCols);
  if (kTopk && !sm.abort) {
    if (warp >= 2 && hist_q >= 0) flush_hist(a, sm, hist_q, tid - 64);
    topk_phase(a, sm, total, g0, g1, sc_cache);
  }
}

// csa_index_scores: sized so that exactly two CTAs share an SM (at most
// 113 KB each): their two 256-column TMEM allocations then always fit the
// SM's 512 columns.
constexpr size_t kSmemPlain = 128 + kSmemHead + (size_t)kStagesPlain * kTileBytes;
static_assert(kSmemPlain <= 112 * 1024, "two CTAs must share an SM");
// csa_index_topk: one CTA per SM, deeper stages and the score cache.
constexpr size_t kSmemFused = 128 + kSmemHead + (size_t)kStagesFused * kTileBytes + (size_t)kScoreCache * 4;
static_assert(kSmemFused <= 227 * 1024, "the fused kernel's shared memory exceeds one CTA's limit");
static_assert((size_t)kCandCap * 8 + 2 * (size_t)kBitmapWords * 4 <= (size_t)kStagesFused * kTileBytes,
              "the selection's candidates and bitmaps must fit the tile stages");

size_t index_tc_smem_bytes() { return kSmemPlain > 80 * 1024 ? kSmemPlain : 80 * 1024; }

cudaError_t launch_index_tc(const Layout& L, int layer, int n, const int32_t* req_ids, const float* q_idx,
                            const float* w, float* scores, int64_t ld, int32_t* n_valid, int ctas,
                            cudaStream_t st, int q_per_req) {
  static std::atomic<uint64_t> attr_set{0};     // devices whose kernel attribute is set
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (setup_needed(attr_set, dev)) {
    e = cudaFuncSetAttribute(index_tc_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             (int)index_tc_smem_bytes());
    if (e != cudaSuccess) return e;
    setup_done(attr_set, dev);
  }
  IndexTcArgs a{L, layer, n, req_ids, q_idx, w, scores, ld, n_valid};
  a.q_per_req = q_per_req;
  index_tc_kernel<false><<<ctas, kThreads, index_tc_smem_bytes(), st>>>(a);
  note_launch();
  return cudaGetLastError();
}

// Workspace of the fused index + top-k: counters and histograms (cleared
// before every launch), per-window candidate counts and the candidate buffer.
struct TopkWs {
  int64_t hist_done, cand_done, qcount, hist, hist2, cand, zero_bytes, total;
};

static TopkWs topk_ws(int n, int64_t ld) {
  auto al = [](int64_t x) { return (x + 255) / 256 * 256; };
  TopkWs w{};
  w.hist_done = 0;
  w.cand_done = al(4LL * n);
  w.qcount = w.cand_done + al(4LL * n);
  w.hist = w.qcount + al(4LL * n);
  w.hist2 = w.hist + al(4LL * n * kHistBins);
  w.zero_bytes = w.hist2 + al(4LL * n * 2048);
  w.cand = w.zero_bytes;
  w.total = w.cand + al(8LL * n * ld);
  return w;
}

size_t index_topk_workspace_bytes(int n, int64_t ld) { return (size_t)topk_ws(n, ld).total; }

// The fused kernel runs one CTA per SM (it allocates TMEM, and its CTAs wait
// for one another, so the launch must fit the resident count the runtime
// guarantees), which leaves room for the score cache.
static size_t index_topk_smem_bytes() { return kSmemFused; }

int index_topk_max_ctas() { return kThreads; }

cudaError_t launch_index_topk(const Layout& L, int layer, int n, const int32_t* req_ids, const float* q_idx,
                              const float* w, float* scores, int64_t ld, int32_t* n_valid, int k, int32_t* idx_out,
                              void* ws, int ctas, cudaStream_t st) {
  // CTAs per SM that can be resident together, per device (the attributes
  // are set and the occupancy asked once on each device)
  static std::atomic<int> occ_by_dev[64];
  int dev = 0, sms = 0;
  cudaError_t e0 = cudaGetDevice(&dev);
  if (e0 == cudaSuccess) e0 = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e0 != cudaSuccess) return e0;
  int occ = dev >= 0 && dev < 64 ? occ_by_dev[dev].load(std::memory_order_acquire) : 0;
  if (occ == 0) {
    cudaError_t e = cudaFuncSetAttribute(index_tc_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)index_topk_smem_bytes());
    if (e == cudaSuccess)
      e = cudaFuncSetAttribute(index_tc_kernel<true>, cudaFuncAttributePreferredSharedMemoryCarveout,
                               (int)cudaSharedmemCarveoutMaxShared);
    if (e == cudaSuccess)
      e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, index_tc_kernel<true>, kThreads, index_topk_smem_bytes());
    if (e != cudaSuccess) return e;
    if (occ < 1) return cudaErrorInvalidConfiguration;
    if (dev >= 0 && dev < 64) occ_by_dev[dev].store(occ, std::memory_order_release);
  }
  // the CTAs of a query wait for one another, so the grid never exceeds what
  // is resident at once; the selection enumerates a query's CTAs one per thread
  if (ctas > occ * sms) ctas = occ * sms;
  if (ctas > kThreads) ctas = kThreads;
  const TopkWs wl = topk_ws(n, ld);
  char* base = static_cast<char*>(ws);
  cudaError_t e = cudaMemsetAsync(base, 0, (size_t)wl.zero_bytes, st);
  if (e != cudaSuccess) return e;
  IndexTcArgs a{L, layer, n, req_ids, q_idx, w, scores, ld, n_valid, k, idx_out,
                reinterpret_cast<int32_t*>(base + wl.hist_done), reinterpret_cast<int32_t*>(base + wl.cand_done),
                reinterpret_cast<uint32_t*>(base + wl.hist), reinterpret_cast<uint32_t*>(base + wl.hist2),
                reinterpret_cast<int32_t*>(base + wl.qcount), reinterpret_cast<uint2*>(base + wl.cand)};
  // the CTAs of a query wait for one another: all must be resident at once
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(ctas);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = index_topk_smem_bytes();
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, index_tc_kernel<true>, a);
  note_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace csa
