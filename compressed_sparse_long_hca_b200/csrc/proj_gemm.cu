// Batch-invariant projection GEMM on the 5th-generation tensor cores
// (csa_gemm_bf16):  Y[t][o] = sum_k X[t][k] W[o][k], BF16 operands, fp32
// accumulation.
//
// What it serves.  Page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力":
// the hidden state of a token is projected to the compressor's candidates and
// gates, and the query side is projected down to d_c = 1024 and up to the
// multi-head (index) queries; page "深度解读DeepSeek V4 看清Benchmark以外的三个
// 范式创新", section 01, "「精度补偿」的无限套娃游戏": the attention output
// (128 heads x 512) is first projected per group of heads, then to the
// model width.  Page "DeepSeek不惜代价保住它！V4关键特性被挖出来了", section
// "牺牲了什么": these GEMMs must be batch-invariant, which the pages obtain by
// replacing the vendor GEMM with one whose reduction does not depend on the
// batch.
//
// Design (swap AB).  The weight rows are the MMA's M (128 output features
// per tile), the tokens its N, always in chunks of 32 (zero padded), and K
// runs in steps of 64: one 16 KB weight tile (stored pre-packed in the
// no-swizzle K-major core-matrix order: one bulk copy) and the matching
// block of the packed activations per stage.  For a token, every output
// element is the same instruction sequence in every batch: the K order is
// fixed (tiles ascending, four K = 16 MMAs per tile in order) and the
// instruction shape (M = 128, N = 32) never changes; the token's column
// inside its chunk does not enter the arithmetic.
//
// Fixed K split.  A weight with few row tiles cannot fill the SMs; its K
// range is then cut into S parts, S chosen from the weight's shape alone
// (never from the batch).  Each part's CTA writes its fp32 partial; the CTA
// that finishes a row tile last (a counter per row tile) adds the S
// partials in part order and writes the output.  The result is therefore
// still independent of the batch, and of which CTA comes last.
//
// Launch.  The activations are packed by a small kernel first; the GEMM is
// launched with programmatic dependent launch behind it, so its CTAs set up
// and start streaming their first weight tiles (which do not depend on the
// pack) while the pack runs, and wait for it before the first activation
// block is copied.
//
// Groups.  With G groups the weight is block diagonal: the rows of group g
// (n_out / G of them, a multiple of 128) read the activation columns
// [g K/G, (g+1) K/G); the host weight then holds only those columns per row.
//
// Roles per CTA (192 threads): warp 0 issues the bulk copies, warp 1 the
// MMAs (one elected lane), warps 2-5 read the accumulator (one TMEM lane =
// one output feature, columns = tokens) and write the output.  All waits
// are bounded; a stuck pipeline records a timeout and returns.
#include "common.cuh"
#include "gemm_out.cuh"
#include "tc.cuh"

namespace csa {

// Device error word of the GEMM (it is not tied to a cache): first error wins.
__device__ int32_t g_gemm_err[2];

namespace {

constexpr int kGThreads = 192;
constexpr int kRowTile = 128;          // output features per tile (MMA M)
constexpr int kKTile = 64;             // K per stage
constexpr int kTokChunk = 32;          // tokens per MMA (N), fixed
constexpr int kWTileBytes = kRowTile * kKTile * 2;     // 16 KB
constexpr int kMaxTok = 256;           // tokens per call
constexpr int kSmemBudget = 100 * 1024;   // two CTAs per SM


__device__ __forceinline__ void gemm_store(const GemmOut& out, int t, int o, float v) {
  int sg = 0;
  while (sg + 1 < out.n_seg && o >= out.seg_end[sg]) ++sg;
  const int r0 = sg > 0 ? out.seg_end[sg - 1] : 0;
  const int64_t rows = out.seg_end[sg] - r0;
  const int64_t at = (int64_t)t * rows + (o - r0);
  if ((out.bf16_mask >> sg) & 1u) static_cast<uint16_t*>(out.y[sg])[at] = bf16_rn(v);
  else static_cast<float*>(out.y[sg])[at] = v;
}

struct GemmArgs {
  const uint8_t* w;       // packed weight tiles [row_tiles][k_tiles][16 KB]
  const uint8_t* xp;      // packed activations [k_tiles][n_pad rows][64], core-matrix order
  int n_out, k_in, n_tok, n_pad;
  int row_tiles, k_tiles;
  int groups;             // block-diagonal groups (1 = dense)
  int splits;             // fixed K split
  GemmOut out;
  float* part;            // [splits][n_tok][n_out] fp32 partials (splits > 1)
  int32_t* done;          // [row_tiles] parts finished (splits > 1; zeroed by the pack kernel)
};

__host__ __device__ __forceinline__ int gemm_stages(int n_pad) {
  const int st = kSmemBudget / (kWTileBytes + n_pad * 128);
  return st > 8 ? 8 : (st < 2 ? 2 : st);
}

}  // namespace

// Pack the columns of X (BF16 [n_tok][row_len]) into the per-k-tile blocks
// the MMA's B operand reads, one group per grid row y (the group's columns
// start at y * kg): block b of a group holds rows 0 .. n_pad-1 of its
// columns [64 b, 64 b + 64), 16-byte chunk c of row t at
// (t/8)*1024 + c*128 + (t%8)*16.  Rows >= n_tok and columns >= kg are zero.
// Also clears the GEMM's row-tile counters (n_done of them, may be null).
__global__ void gemm_pack_x_strided_kernel(const uint16_t* x, int n_tok, int kg, int row_len, int n_pad, int k_tiles,
                                           uint8_t* xp, int32_t* done, int n_done) {
  tc::griddep_launch_dependents();      // the GEMM may become resident now; it waits for this grid's writes
  if (done != nullptr && blockIdx.x == 0 && blockIdx.y == 0)
    for (int u = threadIdx.x; u < n_done; u += blockDim.x) done[u] = 0;
  x += (int64_t)blockIdx.y * kg;
  xp += (int64_t)blockIdx.y * k_tiles * n_pad * 128;
  const int64_t total = (int64_t)k_tiles * n_pad * 8;
  for (int64_t u = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; u < total; u += (int64_t)gridDim.x * blockDim.x) {
    const int c = (int)(u % 8);
    const int t = (int)((u / 8) % n_pad);
    const int b = (int)(u / (8 * (int64_t)n_pad));
    const int k0 = b * kKTile + c * 8;
    uint32_t w4[4] = {0, 0, 0, 0};
    if (t < n_tok)
      for (int q = 0; q < 8; ++q) {
        const uint32_t e = k0 + q < kg ? x[(int64_t)t * row_len + k0 + q] : 0u;
        w4[q >> 1] |= e << (16 * (q & 1));
      }
    *reinterpret_cast<uint4*>(xp + (int64_t)b * n_pad * 128 + (t / 8) * 1024 + c * 128 + (t % 8) * 16) =
        make_uint4(w4[0], w4[1], w4[2], w4[3]);
  }
}

// grid (row_tiles, splits)
__global__ void __launch_bounds__(kGThreads, 2) gemm_bf16_kernel(GemmArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int S = gemm_stages(a.n_pad);
  const int xb = a.n_pad * 128;                      // bytes of one packed activation block
  const int stage_bytes = kWTileBytes + xb;
  uint64_t* full = reinterpret_cast<uint64_t*>(sm + (int64_t)S * stage_bytes);
  uint64_t* empty = full + 8;
  uint64_t* acc_full = empty + 8;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* last_flag = abort_flag + 1;
  const int rt = blockIdx.x, sp = blockIdx.y;
  // this CTA's K tiles (fixed split) and, for a grouped weight, the
  // activation blocks its rows read
  const int kt0 = (int)((int64_t)a.k_tiles * sp / a.splits), kt1 = (int)((int64_t)a.k_tiles * (sp + 1) / a.splits);
  const int rows_per_group = a.n_out / a.groups;
  const int grp = (rt * kRowTile) / rows_per_group;
  const int xblk0 = grp * a.k_tiles;                 // first activation block of the group
  uint32_t ncols = 32;
  while ((int)ncols < a.n_pad) ncols <<= 1;
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, ncols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    for (int s = 0; s < S; ++s) { tc::mbar_init(&full[s], 1); tc::mbar_init(&empty[s], 1); }
    tc::mbar_init(acc_full, 1);
    *abort_flag = 0;
    tc::fence_mbar_init();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int nk = kt1 - kt0;
  bool ok = true;
  int issued = 0;                                    // producer: stages filled so far
  if (warp != 0) tc::griddep_wait();                 // the pack kernel's writes (activations, counters)
  if (warp == 0) {
    // ---- producer: weight tile + activation block per stage.  The weight
    //      tiles of the first stages do not depend on the pack kernel and
    //      are issued before waiting for it.
    const int pre = nk < S ? nk : S;
    if (tc::elect_one()) {
      for (int x = 0; x < pre; ++x) {
        tc::mbar_arrive_expect_tx(&full[x], (uint32_t)stage_bytes);
        tc::bulk_g2s(sm + (int64_t)x * stage_bytes, a.w + ((int64_t)rt * a.k_tiles + kt0 + x) * kWTileBytes,
                     kWTileBytes, &full[x]);
      }
    }
    __syncwarp();
    tc::griddep_wait();
    if (tc::elect_one()) {
      for (int x = 0; x < pre; ++x)
        tc::bulk_g2s(sm + (int64_t)x * stage_bytes + kWTileBytes, a.xp + (int64_t)(xblk0 + kt0 + x) * xb,
                     (uint32_t)xb, &full[x]);
    }
    __syncwarp();
    issued = pre;
    for (int x = pre; x < nk && ok; ++x) {
      const int s = x % S;
      if (x >= S) ok = tc::mbar_wait(&empty[s], ((x / S) - 1) & 1, 1000000000ull);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const int kt = kt0 + x;
      if (tc::elect_one()) {
        uint8_t* st = sm + (int64_t)s * stage_bytes;
        tc::mbar_arrive_expect_tx(&full[s], (uint32_t)stage_bytes);
        tc::bulk_g2s(st, a.w + ((int64_t)rt * a.k_tiles + kt) * kWTileBytes, kWTileBytes, &full[s]);
        tc::bulk_g2s(st + kWTileBytes, a.xp + (int64_t)(xblk0 + kt) * xb, (uint32_t)xb, &full[s]);
      }
      __syncwarp();
      issued = x + 1;
    }
    if (!ok) *abort_flag = 1;
  } else if (warp == 1) {
    // ---- MMA issuer: per K tile, per token chunk, four K = 16 steps in order
    const uint32_t idesc = tc::idesc_bf16(kRowTile, kTokChunk, false, false);
    for (int x = 0; x < nk && ok; ++x) {
      const int s = x % S;
      ok = __all_sync(0xffffffffu, tc::mbar_wait(&full[s], (x / S) & 1, 1000000000ull) && !*abort_flag);
      if (!ok) break;
      tc::tc_fence_after();
      const uint32_t wb = tc::smem_u32(sm + (int64_t)s * stage_bytes), xbase = wb + kWTileBytes;
      if (tc::elect_one()) {
        for (int tc_ = 0; tc_ < a.n_pad / kTokChunk; ++tc_)
          for (int m = 0; m < kKTile / 16; ++m)
            tc::mma_bf16(tmem + kTokChunk * tc_, tc::smem_desc(wb + m * 256, 128, 1024),
                         tc::smem_desc(xbase + tc_ * 4096 + m * 256, 128, 1024), idesc, (x > 0 || m > 0) ? 1u : 0u);
        tc::mma_commit(&empty[s]);
      }
      __syncwarp();
    }
    if (ok) {
      if (tc::elect_one()) tc::mma_commit(acc_full);
      __syncwarp();
    } else {
      *abort_flag = 1;
    }
  } else {
    // ---- epilogue: thread = one output feature (TMEM lane), 16 tokens per load
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;
    const int o = rt * kRowTile + r;
    ok = tc::mbar_wait(acc_full, 0, 1000000000ull) && !*abort_flag;
    if (ok && nk > 0) {
      tc::tc_fence_after();
      for (int c0 = 0; c0 < a.n_pad; c0 += 16) {
        uint32_t v[16];
        tc::tmem_ld_x16(tmem + ((uint32_t)(q4 * 32) << 16) + c0, v);
        tc::tmem_wait_ld();
        if (o < a.n_out) {
          for (int e = 0; e < 16; ++e) {
            const int t = c0 + e;
            if (t >= a.n_tok) break;
            const float y = __uint_as_float(v[e]);
            if (a.splits > 1) a.part[((int64_t)sp * a.n_tok + t) * a.n_out + o] = y;
            else gemm_store(a.out, t, o, y);
          }
        }
      }
    }
    if (a.splits > 1) {
      // the last of the row tile's S CTAs adds the partials in part order
      // (every CTA takes part, also after an abort, so the count completes)
      __threadfence();
      tc::named_bar_sync(1, 128);
      if (tid == 64) last_flag[0] = atomicAdd(&a.done[rt], 1) == a.splits - 1 ? 1 : 0;
      tc::named_bar_sync(1, 128);
      if (last_flag[0] && ok && !*abort_flag) {
        __threadfence();
        if (o < a.n_out) {
          // acc = part 0, then + part 1, + part 2, ...; the loads of up to
          // 16 parts are in flight together
          const int64_t n = (int64_t)a.n_tok * a.n_out;
          for (int t = 0; t < a.n_tok; ++t) {
            const float* p = a.part + (int64_t)t * a.n_out + o;
            float acc = 0.f;
            for (int q0 = 0; q0 < a.splits; q0 += 16) {
              float v[16];
#pragma unroll
              for (int j = 0; j < 16; ++j) v[j] = q0 + j < a.splits ? __ldcg(p + (q0 + j) * n) : 0.f;
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (q0 + j < a.splits) acc = q0 + j == 0 ? v[j] : acc + v[j];
            }
            gemm_store(a.out, t, o, acc);
          }
        }
      }
    }
    if (!ok) *abort_flag = 1;
  }
  tc::tc_fence_before();
  __syncthreads();
  if (*abort_flag && tid == 0) {
    if (atomicCAS(&g_gemm_err[0], 0, (int32_t)kErrTimeout) == 0) g_gemm_err[1] = rt;
    // let the copies already issued land before the shared memory goes away
    for (int x = issued > S ? issued - S : 0; x < issued; ++x) tc::mbar_wait(&full[x % S], (x / S) & 1, 200000000ull);
  }
  if (warp == 1) {
    // no MMA of this CTA is in flight when TMEM is released (the accumulator
    // barrier covers every MMA issued; after an abort, wait on it bounded)
    tc::mbar_wait(acc_full, 0, 200000000ull);
    tc::tmem_dealloc(tmem, ncols);
  }
}

// ---- host side

int gemm_row_tiles(int n_out) { return (n_out + kRowTile - 1) / kRowTile; }
int gemm_k_tiles(int k_in, int groups) { return (k_in / groups + kKTile - 1) / kKTile; }
size_t gemm_weight_bytes(int n_out, int k_in, int groups) {
  return (size_t)gemm_row_tiles(n_out) * gemm_k_tiles(k_in, groups) * kWTileBytes;
}
int gemm_max_tokens() { return kMaxTok; }

// K parts of a weight: as many as keep every CTA resident at once (two per
// SM), each part at least 4 K tiles.  A function of the weight's shape (and
// the device) only.
int gemm_splits(int n_out, int k_in, int groups, int sms) {
  const int rt = gemm_row_tiles(n_out), kt = gemm_k_tiles(k_in, groups);
  int s = 2 * sms / rt;
  if (s > kt / 4) s = kt / 4;
  return s < 1 ? 1 : s;
}

size_t gemm_workspace_bytes(int n_out, int k_in, int groups, int n_tok, int sms) {
  const int n_pad = (n_tok + kTokChunk - 1) / kTokChunk * kTokChunk;
  const size_t xp = (size_t)gemm_k_tiles(k_in, groups) * groups * n_pad * 128;
  const int S = gemm_splits(n_out, k_in, groups, sms);
  const size_t part = S > 1 ? (size_t)S * n_tok * n_out * 4 : 0;
  const size_t done = S > 1 ? (size_t)gemm_row_tiles(n_out) * 4 : 0;
  return (xp + 255) / 256 * 256 + part + done;
}

// Row-major BF16 weight [n_out][k_in] (host) -> packed tiles (host buffer):
// tile (rt, kt) holds rows 128 rt .. 128 rt + 127 and, within the row's
// group, columns 64 kt .. 64 kt + 63; element (r, c) of the tile at
// (r/8)*1024 + (c/8)*128 + (r%8)*16 + (c%8)*2.
void gemm_pack_weight_host(const uint16_t* w, int n_out, int k_in, int groups, uint8_t* dst) {
  const int rt_n = gemm_row_tiles(n_out), kt_n = gemm_k_tiles(k_in, groups);
  const int kg = k_in / groups;
  for (int rt = 0; rt < rt_n; ++rt)
    for (int kt = 0; kt < kt_n; ++kt) {
      uint8_t* tile = dst + ((size_t)rt * kt_n + kt) * kWTileBytes;
      for (int r = 0; r < kRowTile; ++r) {
        const int o = rt * kRowTile + r;
        for (int c = 0; c < kKTile; ++c) {
          const int kk = kt * kKTile + c;
          const uint16_t v = (o < n_out && kk < kg) ? w[(size_t)o * kg + kk] : 0;
          uint8_t* e = tile + (r / 8) * 1024 + (c / 8) * 128 + (r % 8) * 16 + (c % 8) * 2;
          e[0] = (uint8_t)(v & 0xFF);
          e[1] = (uint8_t)(v >> 8);
        }
      }
    }
}

cudaError_t launch_gemm_bf16(const void* w_packed, int n_out, int k_in, int groups, const uint16_t* x, int n_tok,
                             const GemmOut& out, void* ws, int sms, cudaStream_t st) {
  const int n_pad = (n_tok + kTokChunk - 1) / kTokChunk * kTokChunk;
  const int kt = gemm_k_tiles(k_in, groups), rt = gemm_row_tiles(n_out);
  const int S = gemm_splits(n_out, k_in, groups, sms);
  uint8_t* xp = static_cast<uint8_t*>(ws);
  const size_t xp_bytes = ((size_t)kt * groups * n_pad * 128 + 255) / 256 * 256;
  float* part = S > 1 ? reinterpret_cast<float*>(xp + xp_bytes) : nullptr;
  int32_t* done = S > 1 ? reinterpret_cast<int32_t*>(part + (size_t)S * n_tok * n_out) : nullptr;
  // packed activations: group g's k tiles are blocks g kt .. g kt + kt - 1
  cudaError_t e = cudaSuccess;
  {
    const int kg = k_in / groups;
    const int64_t chunks = (int64_t)kt * n_pad * 8;
    const int blocks = (int)((chunks + 255) / 256 < 2048 ? (chunks + 255) / 256 : 2048);
    gemm_pack_x_strided_kernel<<<dim3(blocks, groups), 256, 0, st>>>(x, n_tok, kg, k_in, n_pad, kt, xp, done, rt);
    note_launch();
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  const size_t smem = (size_t)gemm_stages(n_pad) * (kWTileBytes + n_pad * 128) + 256 + 128;
  static std::atomic<uint64_t> attr_set{0};     // devices whose kernel attributes are set
  int dev = 0;
  e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (setup_needed(attr_set, dev)) {
    e = cudaFuncSetAttribute(gemm_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(gemm_bf16_kernel, cudaFuncAttributePreferredSharedMemoryCarveout, 100);
    if (e != cudaSuccess) return e;
    setup_done(attr_set, dev);
  }
  GemmArgs a{static_cast<const uint8_t*>(w_packed), xp, n_out, k_in, n_tok, n_pad, rt, kt, groups, S, out, part,
             done};
  cudaLaunchConfig_t lc{};
  lc.gridDim = dim3(rt, S);
  lc.blockDim = dim3(kGThreads);
  lc.dynamicSmemBytes = smem;
  lc.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = at;
  lc.numAttrs = 1;
  e = cudaLaunchKernelEx(&lc, gemm_bf16_kernel, a);
  note_launch();
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

// Read and clear the GEMM's device error word (synchronises `st`).
cudaError_t gemm_read_error(int32_t* code, int32_t* detail, cudaStream_t st) {
  cudaError_t e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return e;
  int32_t w[2] = {0, 0};
  e = cudaMemcpyFromSymbol(w, g_gemm_err, sizeof w);
  if (e != cudaSuccess) return e;
  *code = w[0];
  *detail = w[1];
  if (w[0] != 0) {
    const int32_t z[2] = {0, 0};
    e = cudaMemcpyToSymbol(g_gemm_err, z, sizeof z);
  }
  return e;
}

}  // namespace csa
