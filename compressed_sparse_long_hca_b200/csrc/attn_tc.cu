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
// Per query the rows are: selected entries (ascending; HCA: all entries)
// then the window (ascending positions); K = V = the stored row.  Because
// the KV head is shared, QK^T and PV are dense products.  A CTA owns one
// query and a group of G heads and walks the rows in tiles of 128:
//   * all threads gather the tile's rows from the paged cache and the ring,
//     dequantise them to BF16 and store them in shared memory in the
//     no-swizzle core-matrix order;
//   * QK: S^T[128 rows x G heads] = K_tile Q^T on tcgen05 (kind::f16,
//     M = 128 rows, N = G heads, K = 16 dims per instruction) into TMEM;
//   * softmax: one thread per row reads its G logits; per-head maxima and
//     sums go through shared memory in a fixed order.  The running maximum
//     of a head is only raised when a tile exceeds it by more than 8 (then
//     the head's accumulator column is rescaled), so most tiles need no
//     rescale; every decision depends on the query's own data only;
//   * PV: O^T[dims x G] += V_tile^T P^T on tcgen05, the same shared-memory
//     tile read as an MN-major A operand, P^T (BF16) as an MN-major B operand;
//   * the sink enters at the end: out = O e^{m-mu} / (l e^{m-mu} + e^{sink-mu}),
//     mu = max(m, sink).
// A query's reduction over rows is never split across CTAs.  Launch
// variants differ only in G (heads per CTA); every per-head operation is
// independent of G, so the variants return identical bits.
#include "common.cuh"
#include "tc.cuh"

namespace csa {

namespace {

constexpr int kAttThreads = 256;       // warps 0-3: TMEM lanes / softmax; all: gather
constexpr int kTileRows = 128;
constexpr float kSlack = 8.f;          // stale running maximum allowed below a tile's max
constexpr int kMaxK = 8192;

struct AttnTcArgs {
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
  int G;            // heads per CTA (MMA N), 16 or 32
};

struct AttnSmemLayout {
  int Dp;           // head dim padded to a multiple of 128
  int64_t tile, qs, pt, stage, sel, rsc, stats, bars, total;
};

__host__ __device__ inline AttnSmemLayout attn_smem_layout(int D, int G, int k) {
  AttnSmemLayout s{};
  s.Dp = (D + 127) / 128 * 128;
  int64_t o = 0;
  s.tile = o;  o += (int64_t)kTileRows * s.Dp * 2;           // BF16 rows, core-matrix order
  s.qs = o;    o += (int64_t)G * s.Dp * 2;                   // BF16 query heads
  s.pt = o;    o += (int64_t)kTileRows * G * 2 * 2;          // BF16 P^T and (P*scale)^T (MN-major)
  s.stage = o; o += (int64_t)kTileRows * (G + 1) * 4;        // fp32 logits / p for reductions
  s.sel = o;   o += (int64_t)(k > 0 ? k : 1) * 4;            // compacted selected entries
  s.rsc = o;   o += (int64_t)kTileRows * 4;                  // per-row FP8 scale of the tile
  o = (o + 15) / 16 * 16;
  s.stats = o; o += (int64_t)(6 * 32 + 4 * 32) * 4;          // m, l, corr, mt, den, cm; partials [4][32]
  o = (o + 15) / 16 * 16;
  s.bars = o;  o += 64;
  s.total = o;
  return s;
}

}  // namespace

__global__ void __launch_bounds__(kAttThreads, 1) attn_tc_kernel(AttnTcArgs a) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const Layout& L = a.L;
  const int D = L.D, R = L.R, H = L.H, G = a.G;
  const AttnSmemLayout S = attn_smem_layout(D, G, a.k);
  const int Dp = S.Dp;
  const uint32_t sbo_rows = (uint32_t)Dp * 16;        // bytes between 8-row groups of the tile
  uint8_t* tile = sm + S.tile;
  uint8_t* qs = sm + S.qs;
  uint8_t* pt = sm + S.pt;
  float* stage = reinterpret_cast<float*>(sm + S.stage);
  int32_t* sel = reinterpret_cast<int32_t*>(sm + S.sel);
  float* rsc = reinterpret_cast<float*>(sm + S.rsc);
  uint8_t* ptm = pt + kTileRows * G * 2;                   // (P * row scale)^T for the FP8 dims
  float* m_run = reinterpret_cast<float*>(sm + S.stats);
  float* l_run = m_run + 32;
  float* corr = l_run + 32;
  float* m_tile = corr + 32;
  float* den = m_tile + 32;
  float* cmul = den + 32;
  float* part = cmul + 32;                                  // [4][32]
  uint64_t* bar_qk = reinterpret_cast<uint64_t*>(sm + S.bars);
  uint64_t* bar_pv = bar_qk + 1;
  uint64_t* bar_drain = bar_qk + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_qk + 3);
  __shared__ int s_nsel, s_flag;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int i = blockIdx.x;
  const int h0 = blockIdx.y * G;
  const int req = a.req_ids[i];
  if (req < 0 || req >= L.max_req) {
    if (tid == 0 && blockIdx.y == 0) set_err(L, kErrBounds, i);
    return;
  }
  const bool csa = a.layer < L.n_csa;
  const int64_t T = L.lengths()[(int64_t)a.layer * L.max_req + req];
  if (T <= 0) {
    if (tid == 0 && blockIdx.y == 0) set_err(L, kErrBounds, 1000000 + i);
    return;
  }
  const int64_t t = T - 1;
  const int64_t n_entries = csa ? T / kCsaM : T / kHcaM;
  const int64_t w0 = t - (kWindow - 1) > 0 ? t - (kWindow - 1) : 0;
  const int64_t n_win = t - w0 + 1;

  // ---- set-up: TMEM (S^T: G columns, O^T: Dp/128 chunks of G columns), barriers
  if (warp == 0) {
    tc::tmem_alloc(tmem_slot, 256);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    tc::mbar_init(bar_qk, 1);
    tc::mbar_init(bar_pv, 1);
    tc::mbar_init(bar_drain, 1);
    tc::fence_mbar_init();
  }
  if (tid < 32) { m_run[tid] = -INFINITY; l_run[tid] = 0.f; }
  // compact the selected list (CSA) in order, dropping -1 and out-of-range entries
  int64_t n_sel = csa ? 0 : n_entries;
  if (csa) {
    if (tid == 0) s_nsel = 0;
    __syncthreads();
    for (int base = 0; base < a.k; base += kAttThreads) {
      const int x = base + tid;
      int j = x < a.k ? a.topk[(int64_t)i * a.k + x] : -1;
      if (j >= n_entries) { set_err(L, kErrBounds, 2000000 + i); j = -1; }
      const int v = j >= 0 ? 1 : 0;
      // ordered compaction of this chunk of 256
      const unsigned ballot = __ballot_sync(0xffffffffu, v);
      const int wcount = __popc(ballot);
      const int wpre = __popc(ballot & ((1u << lane) - 1));
      __syncthreads();
      if (lane == 0) part[warp] = (float)wcount;            // reuse as scratch (counts < 2^24)
      __syncthreads();
      int before = s_nsel;
      for (int w = 0; w < warp; ++w) before += (int)part[w];
      if (v) sel[before + wpre] = j;
      __syncthreads();
      if (tid == 0) {
        int tot = 0;
        for (int w = 0; w < kAttThreads / 32; ++w) tot += (int)part[w];
        s_nsel += tot;
      }
    }
    __syncthreads();
    n_sel = s_nsel;
  }
  // cos/sin of the query position for each RoPE pair, shared by all heads
  float2* cs = reinterpret_cast<float2*>(stage);
  for (int p = tid; p < R / 2; p += kAttThreads) {
    float c = 1.f, sn = 0.f;
    rope_pair(c, sn, L.theta()[p], t);      // rotating (1, 0) gives (cos, sin)
    cs[p] = make_float2(c, sn);
  }
  __syncthreads();
  // query heads h0 .. h0+G-1, rotated at t, as BF16 in K-major core-matrix order
  for (int x = tid; x < G * (Dp / 8); x += kAttThreads) {
    const int hh = x / (Dp / 8), c = x % (Dp / 8);
    const int h = h0 + hh;
    uint32_t pk[4] = {0, 0, 0, 0};
    if (h < H) {
      const uint16_t* qh = a.q + ((int64_t)i * H + h) * D;
      float v[8];
      for (int e = 0; e < 8; ++e) v[e] = (8 * c + e < D) ? bf16_val(qh[8 * c + e]) : 0.f;
      if (8 * c >= D - R && 8 * c < D) {
        for (int e = 0; e < 8; e += 2) {
          const float2 w = cs[(8 * c + e - (D - R)) / 2];
          const float x0 = v[e], x1 = v[e + 1];
          v[e] = x0 * w.x - x1 * w.y;
          v[e + 1] = x0 * w.y + x1 * w.x;
        }
      }
      for (int e = 0; e < 4; ++e) pk[e] = (uint32_t)bf16_rn(v[2 * e]) | ((uint32_t)bf16_rn(v[2 * e + 1]) << 16);
    }
    *reinterpret_cast<uint4*>(qs + (hh >> 3) * sbo_rows + c * 128 + (hh & 7) * 16) =
        make_uint4(pk[0], pk[1], pk[2], pk[3]);
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
  // TMEM columns: S_fp8 (logit part over the FP8 dims, before the row
  // scale), S_bf16 (RoPE dims), then per 128-dim chunk of the output an
  // accumulator for the FP8 dims (B = (P*scale)^T) and, where the chunk
  // holds RoPE dims, one for those (B = P^T).
  const uint32_t col_s = 0, col_sr = 32, col_o = 64;
  const int n_dc = Dp / 128;
  const int dmain = D - R;
  const int dc_r0 = dmain / 128;                            // first chunk holding RoPE dims
  const int64_t total = n_sel + n_win;
  const int n_tiles = (int)((total + kTileRows - 1) / kTileRows);
  const char* st_ring = L.state(req, a.layer);
  const uint32_t id_qk = tc::idesc_bf16(128, G, false, false);
  const uint32_t id_pv = tc::idesc_bf16(128, G, true, true);
  bool ok = true;

  for (int tt = 0; tt < n_tiles && ok; ++tt) {
    // -- the previous tile's PV has finished: tile and P^T buffers are free
    if (tt > 0) ok = tc::mbar_wait(bar_pv, (tt - 1) & 1);
    ok = __syncthreads_and(ok) != 0;
    if (!ok) break;
    tc::tc_fence_after();
    // -- gather + dequantise: thread handles row (tid % 128), half of the chunks
    {
      const int r = tid & (kTileRows - 1);
      const int64_t rr = (int64_t)tt * kTileRows + r;
      const uint8_t* f8 = nullptr;
      const uint16_t* bf = nullptr;
      float sc = 0.f;
      if (rr < n_sel) {
        const int64_t j = csa ? (int64_t)sel[rr] : rr;
        const float* scp;
        L.entry_row(req, a.layer, j, &f8, &bf, &scp);
        sc = *scp;
      } else if (rr < total) {
        const int slot = (int)((w0 + (rr - n_sel)) % kWindow);
        f8 = reinterpret_cast<const uint8_t*>(st_ring + L.ring_fp8) + (int64_t)slot * (D - R);
        bf = reinterpret_cast<const uint16_t*>(st_ring + L.ring_bf16) + (int64_t)slot * R;
        sc = reinterpret_cast<const float*>(st_ring + L.ring_scale)[slot];
      }
      if (tid < kTileRows) rsc[r] = sc;
      // This thread covers dims [lo, hi) of the row.  Issue every global load
      // first (16-byte units: 16 FP8 dims or 8 BF16 dims), then convert.
      const int lo = (tid >> 7) * (Dp / 2), hi = lo + Dp / 2;
      const int f_lo = lo < D - R ? lo : D - R, f_hi = hi < D - R ? hi : D - R;          // FP8 dims
      const int r_lo = lo > D - R ? (lo < D ? lo : D) : D - R, r_hi = hi < D ? hi : D;   // RoPE dims
      const int nf = f_hi > f_lo ? (f_hi - f_lo) / 16 : 0;
      const int nr = r_hi > r_lo ? (r_hi - r_lo) / 8 : 0;
      constexpr int kMaxUnits = 24;
      uint4 buf[kMaxUnits];
#pragma unroll
      for (int x = 0; x < kMaxUnits; ++x) {
        buf[x] = make_uint4(0, 0, 0, 0);
        if (f8 != nullptr) {
          if (x < nf) buf[x] = *reinterpret_cast<const uint4*>(f8 + f_lo + 16 * x);
          else if (x < nf + nr) buf[x] = *reinterpret_cast<const uint4*>(bf + (r_lo - (D - R)) + 8 * (x - nf));
        }
      }
      uint8_t* dst = tile + (r >> 3) * sbo_rows + (r & 7) * 16;
#pragma unroll
      for (int x = 0; x < kMaxUnits; ++x) {
        if (x < nf) {   // 16 FP8 values -> two 8-dim BF16 chunks (exact conversion)
          const uint32_t wv[4] = {buf[x].x, buf[x].y, buf[x].z, buf[x].w};
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const uint32_t b2 = (wv[e >> 1] >> (16 * (e & 1))) & 0xFFFFu;
            const __half2_raw h2 = __nv_cvt_fp8x2_to_halfraw2((__nv_fp8x2_storage_t)b2, __NV_E4M3);
            const float2 f = __half22float2(__half2(h2));
            pk[e] = (uint32_t)bf16_rn(f.x) | ((uint32_t)bf16_rn(f.y) << 16);
          }
          const int c = (f_lo + 16 * x) / 8;
          *reinterpret_cast<uint4*>(dst + c * 128) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          *reinterpret_cast<uint4*>(dst + (c + 1) * 128) = make_uint4(pk[4], pk[5], pk[6], pk[7]);
        } else if (x < nf + nr) {
          const int c = (r_lo + 8 * (x - nf)) / 8;
          *reinterpret_cast<uint4*>(dst + c * 128) = buf[x];
        }
      }
      // dims past D (padding up to a multiple of 128) are zero
      for (int c = (D > lo ? (D < hi ? D : hi) : lo) / 8; c < hi / 8; ++c)
        *reinterpret_cast<uint4*>(dst + c * 128) = make_uint4(0, 0, 0, 0);
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
          const bool main = 16 * ks < dmain;                  // (D - R) is a multiple of 16
          const int k0 = main ? 0 : dmain / 16;
          tc::mma_bf16(tmem + (main ? col_s : col_sr), tc::smem_desc(ta + ks * 256, 128, sbo_rows),
                       tc::smem_desc(tq + ks * 256, 128, sbo_rows), id_qk, ks > k0 ? 1u : 0u);
        }
        tc::mma_commit(bar_qk);
      }
      __syncwarp();
    }
    // -- softmax statistics (warps 0-3 own the 128 TMEM lanes = rows)
    const int r = tid;                       // valid for warps 0-3
    const int64_t rr = (int64_t)tt * kTileRows + r;
    float u[32];
    if (warp < 4) {
      ok = tc::mbar_wait(bar_qk, tt & 1);
      tc::tc_fence_after();
      uint32_t sv[32], sr[32];
      tc::tmem_ld_x16(tmem + lane_base + col_s, sv);
      tc::tmem_ld_x16(tmem + lane_base + col_sr, sr);
      if (G > 16) {
        tc::tmem_ld_x16(tmem + lane_base + col_s + 16, sv + 16);
        tc::tmem_ld_x16(tmem + lane_base + col_sr + 16, sr + 16);
      }
      tc::tmem_wait_ld();
      const float rs = rsc[r];
      for (int h = 0; h < 32; ++h) {
        u[h] = (h < G && rr < total)
                   ? fmaf(rs, __uint_as_float(sv[h]), __uint_as_float(sr[h])) * a.scale
                   : -INFINITY;
        if (h < G) stage[r * (G + 1) + h] = u[h];
      }
    }
    ok = __syncthreads_and(ok) != 0;
    if (!ok) break;
    if (warp < 4) {   // warp w, lane h: max over rows 32w .. 32w+31 of head h
      if (lane < G) {
        float mx = -INFINITY;
        for (int x = 0; x < 32; ++x) mx = fmaxf(mx, stage[(warp * 32 + x) * (G + 1) + lane]);
        part[warp * 32 + lane] = mx;
      }
    }
    __syncthreads();
    if (tid < G) {
      const float mt = fmaxf(fmaxf(part[tid], part[32 + tid]), fmaxf(part[64 + tid], part[96 + tid]));
      const float mo = m_run[tid];
      float c = 1.f;
      if (mt > mo + kSlack || (mo == -INFINITY && mt > -INFINITY)) {
        c = (mo == -INFINITY) ? 0.f : expf(mo - mt);
        m_run[tid] = mt;
      }
      corr[tid] = c;
      l_run[tid] *= c;
    }
    if (tid == 0) s_flag = 0;
    __syncthreads();
    if (tid < G && corr[tid] != 1.f && tt > 0) s_flag = 1;
    __syncthreads();
    // -- rescale the accumulator columns of heads whose running max moved
    if (s_flag && warp < 4) {
      for (int dc = 0; dc < n_dc + (n_dc - dc_r0); ++dc) {
        for (int hb = 0; hb < G; hb += 16) {
          uint32_t ov[16];
          const uint32_t addr = tmem + lane_base + col_o + dc * 32 + hb;
          tc::tmem_ld_x16(addr, ov);
          tc::tmem_wait_ld();
          for (int e = 0; e < 16; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * corr[hb + e]);
          tc::tmem_st_x16(addr, ov);
        }
      }
      tc::tmem_wait_st();
    }
    // -- p = exp(u - m_run): P^T (BF16, MN-major) for PV, fp32 copy for the sums
    if (warp < 4) {
      const float rs = rsc[r];
      for (int hg = 0; hg < G / 8; ++hg) {
        uint32_t pk[4], pm[4];
        for (int e = 0; e < 8; e += 2) {
          const int h = hg * 8 + e;
          const float p0 = expf(u[h] - m_run[h]);
          const float p1 = expf(u[h + 1] - m_run[h + 1]);
          stage[r * (G + 1) + h] = p0;
          stage[r * (G + 1) + h + 1] = p1;
          pk[e >> 1] = (uint32_t)bf16_rn(p0) | ((uint32_t)bf16_rn(p1) << 16);
          pm[e >> 1] = (uint32_t)bf16_rn(p0 * rs) | ((uint32_t)bf16_rn(p1 * rs) << 16);
        }
        *reinterpret_cast<uint4*>(pt + hg * 2048 + (r >> 3) * 128 + (r & 7) * 16) =
            make_uint4(pk[0], pk[1], pk[2], pk[3]);
        *reinterpret_cast<uint4*>(ptm + hg * 2048 + (r >> 3) * 128 + (r & 7) * 16) =
            make_uint4(pm[0], pm[1], pm[2], pm[3]);
      }
    }
    tc::fence_proxy_async_smem();
    tc::tc_fence_before();
    __syncthreads();
    tc::tc_fence_after();
    // -- PV: O^T[dims x heads] += V^T P^T
    if (warp == 0) {
      if (tc::elect_one()) {
        const uint32_t ta = tc::smem_u32(tile), tp = tc::smem_u32(pt), tpm = tc::smem_u32(ptm);
        // FP8 dims: chunks 0 .. n_dc-1 with B = (P*scale)^T; RoPE dims: chunks
        // dc_r0 .. n_dc-1 again with B = P^T, into their own accumulators
        for (int x = 0; x < n_dc + (n_dc - dc_r0); ++x) {
          const bool main = x < n_dc;
          const int dc = main ? x : dc_r0 + (x - n_dc);
          for (int ks = 0; ks < kTileRows / 16; ++ks)
            tc::mma_bf16(tmem + col_o + x * 32, tc::smem_desc(ta + dc * 16 * 128 + ks * 2 * sbo_rows, sbo_rows, 128),
                         tc::smem_desc((main ? tpm : tp) + ks * 256, 128, 2048), id_pv, (tt > 0 || ks > 0) ? 1u : 0u);
        }
        tc::mma_commit(bar_pv);
      }
      __syncwarp();
    }
    // -- row sums of p for each head (warp w: rows 32w..32w+31), fixed order
    if (warp < 4 && lane < G) {
      float sum = 0.f;
      for (int x = 0; x < 32; ++x) sum += stage[(warp * 32 + x) * (G + 1) + lane];
      part[warp * 32 + lane] = sum;
    }
    __syncthreads();
    if (tid < G) l_run[tid] += ((part[tid] + part[32 + tid]) + part[64 + tid]) + part[96 + tid];
  }
  // ---- finish: out = O e^{m-mu} / (l e^{m-mu} + e^{sink-mu})
  if (ok && n_tiles > 0) ok = tc::mbar_wait(bar_pv, (n_tiles - 1) & 1);
  ok = __syncthreads_and(ok) != 0;
  if (ok) {
    tc::tc_fence_after();
    if (tid < G) {
      const int h = h0 + tid;
      const float sk = h < H ? a.sink[h] : 0.f;
      const float mf = fmaxf(m_run[tid], sk);
      const float cm = expf(m_run[tid] - mf);
      cmul[tid] = cm;
      den[tid] = l_run[tid] * cm + expf(sk - mf);
    }
    __syncthreads();
    if (warp < 4) {
      for (int dc = 0; dc < n_dc; ++dc) {
        const int d = dc * 128 + tid;
        // FP8 dims read the scaled accumulator, RoPE dims their own.  TMEM
        // loads are warp-collective, so a chunk that holds both kinds loads
        // both and every lane keeps its own.
        const bool has_rope = dc >= dc_r0;
        for (int hb = 0; hb < G; hb += 16) {
          uint32_t om[16], orp[16];
          tc::tmem_ld_x16(tmem + lane_base + col_o + dc * 32 + hb, om);
          if (has_rope) tc::tmem_ld_x16(tmem + lane_base + col_o + (n_dc + dc - dc_r0) * 32 + hb, orp);
          tc::tmem_wait_ld();
          for (int e = 0; e < 16; ++e) {
            const int h = h0 + hb + e;
            const float ov = __uint_as_float(d < dmain ? om[e] : orp[e]);
            if (h < H && d < D)
              a.out[((int64_t)i * H + h) * D + d] = bf16_rn(__fdiv_rn(ov * cmul[hb + e], den[hb + e]));
          }
        }
      }
    }
  } else if (tid == 0) {
    set_err(L, kErrTimeout, 3000000 + i);
  }
  if (warp == 0) {   // no tcgen05 operation of this CTA is in flight when TMEM is released
    if (tc::elect_one()) tc::mma_commit(bar_drain);
    __syncwarp();
    tc::mbar_wait(bar_drain, 0, 200000000ull);
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 0) tc::tmem_dealloc(tmem, 256);
}

size_t attn_tc_smem_bytes(int D, int G, int k) { return (size_t)attn_smem_layout(D, G, k).total + 1024; }

cudaError_t launch_attn_tc(const Layout& L, int layer, int n, const int32_t* req_ids, const uint16_t* q,
                           const int32_t* topk, int k, const float* sink, float scale, uint16_t* out, int G,
                           cudaStream_t st) {
  const size_t sm = attn_tc_smem_bytes(L.D, G, k);
  if (sm > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  AttnTcArgs a{L, layer, n, req_ids, q, topk, k, sink, scale, out, G};
  dim3 grid(n, (L.H + G - 1) / G);
  attn_tc_kernel<<<grid, kAttThreads, sm, st>>>(a);
  return cudaGetLastError();
}

}  // namespace csa
