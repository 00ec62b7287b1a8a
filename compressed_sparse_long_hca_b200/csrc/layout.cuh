// Arena layout of the CSA / HCA cache, shared by the host code and the kernels.
//
// The split into a per-request state cache and a paged classic cache follows
// page "V4终于终于终于终于是来了", section "HCA——重度压缩注意力" (cache
// paragraph): the state cache holds, per request, the latest 128 raw tokens'
// KV and the tails that have not yet filled a 4- or 128-token window; the
// classic cache holds compressed entries in blocks of lcm(4, 128) = 128 raw
// tokens, i.e. 32 CSA entries and 1 HCA entry per block and layer.
//
// Pages: the pool hands out pages of 4 consecutive blocks (512 raw tokens)
// to a request; a page therefore holds, per CSA layer, 128 compressed entries
// and, per HCA layer, 4.  A request's block b lives in page b / 4.
//
// Arena (one caller-owned device buffer, every section 256-byte aligned):
//   header      error word (int32 code, int32 detail, int64 info)
//   tickets     int32 [n_layers][max_req]         CTA tickets of the one-launch append
//   lengths     int64 [n_layers][max_req]         tokens appended so far
//   capacity    int32 [max_req]                   pages held by the request
//   page table  int32 [max_req][max_pages_per_req]  logical -> pool page
//   theta       fp64 [R/2]                        RoPE frequencies
//   b_pos       fp32 [n_csa][8][D], [n_csa][8][d_I], [n_hca][128][D]
//   state       per request, per layer:
//                 window ring: fp8 [128][D-R] | bf16 [128][R] | fp32 [128]
//                 CSA tail:    fp32 c[8][D] | z[8][D] | ci[8][d_I] | zi[8][d_I]
//                 HCA tail:    fp32 c[128][D] | z[128][D]
//   pool        pool_pages x page, page = per layer a section of P rows
//               (P = 128 for CSA, 4 for HCA):
//                 fp8 [P][D-R] | bf16 [P][R] | fp32 scale [P]
//               and for CSA layers the index keys of the page's 128 entries:
//                 codes: 16 groups of 8 keys x CHs 16-byte chunks
//                 scale chunk: 512 bytes of E8M0 scales
//
// Storage formats (one per cache):
//   mixed (the pages' formats): as above.
//   fp32: every stored vector is plain fp32 -- a KV row is D floats (RoPE
//         dims rotated), an index key d_I floats; the ring is [128][D] fp32,
//         a CSA page section [128][D] fp32 rows then [128][d_I] fp32 keys,
//         an HCA page section [4][D] fp32 rows.
//
// Index keys are stored as one ready-made tcgen05 operand tile per page.
// Codes: key s, 16-byte chunk c (32 E2M1 values) at (s/8)*(CHs*128) + c*128 +
// (s%8)*16, the K-major no-swizzle core-matrix order (CHs = d_I/32 rounded up
// to even; padding chunks are zero).  Scales: key s = 32*m1 + m0, its
// scale k at byte 16*m0 + 4*m1 + k (k < 4; missing k hold 127 = 1.0), the
// 32 x 128-bit order that tcgen05.cp copies into the MMA's scale columns.
#pragma once
#include <stddef.h>
#include <stdint.h>

namespace csa {

constexpr int kWindow = 128;      // raw-token window
constexpr int kCsaM = 4;          // CSA compression ratio
constexpr int kCsaWin = 8;        // CSA window (2m, overlapping)
constexpr int kHcaM = 128;        // HCA compression ratio
constexpr int kBlockTokens = 128; // classic-cache block, lcm(4, 128): 32 CSA + 1 HCA entries
constexpr int kCsaPerBlock = 32;
constexpr int kBlocksPerPage = 4;
constexpr int kPageTokens = kBlockTokens * kBlocksPerPage;   // 512
constexpr int kCsaPerPage = kCsaPerBlock * kBlocksPerPage;    // 128 (one MMA tile)
constexpr int kHcaPerPage = kBlocksPerPage;                   // 4
constexpr int kSfChunk = 512;

constexpr int64_t kAlign = 256;
__host__ __device__ constexpr int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

constexpr int kFmtMixed = 0;      // FP8 + BF16 rows, MXFP4 index keys
constexpr int kFmtF32 = 1;        // fp32 rows and index keys

struct Layout {
  // shapes
  int H, D, R, HI, dI, CHs;
  int fmt;                  // kFmtMixed or kFmtF32
  int n_csa, n_hca, n_layers;
  int max_req, max_pages_per_req, pool_pages;
  float rope_base;
  // arena base
  char* base;
  // section offsets from base
  int64_t off_err, off_tick, off_len, off_cap, off_pt, off_theta, off_bkv, off_bidx, off_bhca, off_state, off_pool;
  // row sections
  int64_t kv_fp8_bytes;     // D - R
  int64_t kv_bf16_bytes;    // 2R
  // state sizes
  int64_t ring_fp8, ring_bf16, ring_scale, ring_bytes;          // offsets inside a ring
  int64_t csa_tail_bytes, hca_tail_bytes;
  int64_t state_csa_layer, state_hca_layer, state_req;          // strides
  // page sections (per layer kind)
  int64_t pg_csa_bf16, pg_csa_scale, pg_idx_codes, pg_idx_sf, pg_csa_bytes;
  int64_t pg_hca_bf16, pg_hca_scale, pg_hca_bytes;
  int64_t idx_tile_bytes;   // codes + scale chunk of one page (one bulk copy)
  int64_t pg_idx_f32;       // fp32 format: offset of the index keys in a CSA page section
  int64_t page_bytes;
  int64_t total_bytes;

  __host__ __device__ int64_t* lengths() const { return reinterpret_cast<int64_t*>(base + off_len); }
  __host__ __device__ int32_t* capacity() const { return reinterpret_cast<int32_t*>(base + off_cap); }
  __host__ __device__ int32_t* page_table(int req) const {
    return reinterpret_cast<int32_t*>(base + off_pt) + (int64_t)req * max_pages_per_req;
  }
  __host__ __device__ int32_t* err() const { return reinterpret_cast<int32_t*>(base + off_err); }
  __host__ __device__ int32_t* ticket(int layer, int req) const {
    return reinterpret_cast<int32_t*>(base + off_tick) + (int64_t)layer * max_req + req;
  }
  // RoPE frequencies base^(-2i/R), i < R/2, in fp64 (written at initialisation)
  __host__ __device__ const double* theta() const { return reinterpret_cast<const double*>(base + off_theta); }
  __host__ __device__ const float* bpos_csa(int layer) const {
    return reinterpret_cast<const float*>(base + off_bkv) + (int64_t)layer * kCsaWin * D;
  }
  __host__ __device__ const float* bpos_idx(int layer) const {
    return reinterpret_cast<const float*>(base + off_bidx) + (int64_t)layer * kCsaWin * dI;
  }
  __host__ __device__ const float* bpos_hca(int hlayer) const {
    return reinterpret_cast<const float*>(base + off_bhca) + (int64_t)hlayer * kHcaM * D;
  }
  // state of (request, layer): ring first, then the tail
  __host__ __device__ char* state(int req, int layer) const {
    int64_t o = off_state + (int64_t)req * state_req;
    if (layer < n_csa) o += (int64_t)layer * state_csa_layer;
    else o += (int64_t)n_csa * state_csa_layer + (int64_t)(layer - n_csa) * state_hca_layer;
    return base + o;
  }
  __host__ __device__ char* tail(int req, int layer) const { return state(req, layer) + ring_bytes; }
  // section of pool page `pg` that belongs to `layer`
  __host__ __device__ char* page(int64_t pg, int layer) const {
    int64_t o = off_pool + pg * page_bytes;
    if (layer < n_csa) o += (int64_t)layer * pg_csa_bytes;
    else o += (int64_t)n_csa * pg_csa_bytes + (int64_t)(layer - n_csa) * pg_hca_bytes;
    return base + o;
  }
  __host__ __device__ int rows_per_page(int layer) const { return layer < n_csa ? kCsaPerPage : kHcaPerPage; }
  // stored KV row of compressed entry j of (req, layer)
  __host__ __device__ void entry_row(int req, int layer, int64_t j, const uint8_t** fp8, const uint16_t** bf16,
                                     const float** scale) const {
    const int P = rows_per_page(layer);
    const char* pp = page(page_table(req)[j / P], layer);
    const int s = (int)(j % P);
    const bool csa = layer < n_csa;
    *fp8 = reinterpret_cast<const uint8_t*>(pp) + (int64_t)s * kv_fp8_bytes;
    *bf16 = reinterpret_cast<const uint16_t*>(pp + (csa ? pg_csa_bf16 : pg_hca_bf16)) + (int64_t)s * R;
    *scale = reinterpret_cast<const float*>(pp + (csa ? pg_csa_scale : pg_hca_scale)) + s;
  }
  // fp32 format: stored row of compressed entry j, its index key, a ring row
  __host__ __device__ float* entry_row_f32(int req, int layer, int64_t j) const {
    const int P = rows_per_page(layer);
    return reinterpret_cast<float*>(page(page_table(req)[j / P], layer)) + (j % P) * D;
  }
  __host__ __device__ float* index_key_f32(int req, int layer, int64_t j) const {
    return reinterpret_cast<float*>(page(page_table(req)[j / kCsaPerPage], layer) + pg_idx_f32) +
           (j % kCsaPerPage) * dI;
  }
  __host__ __device__ float* ring_row_f32(int req, int layer, int slot) const {
    return reinterpret_cast<float*>(state(req, layer)) + (int64_t)slot * D;
  }
  // byte offset of chunk c of index key s inside a page's code tile
  __host__ __device__ int64_t idx_code_off(int s, int c) const {
    return (int64_t)(s >> 3) * (CHs * 128) + c * 128 + (s & 7) * 16;
  }
  // byte offset of scale k of index key s inside a page's scale chunk
  __host__ __device__ static int idx_sf_off(int s, int k) { return 16 * (s & 31) + 4 * (s >> 5) + k; }
};

// Counts the kernels libcsa has queued (csa_launch_count).
void note_launch();

// Device error word: first error wins.
enum DevErr : int32_t {
  kErrNone = 0,
  kErrBounds = 1,     // request id / block / index out of range
  kErrCapacity = 2,   // append beyond the request's blocks
  kErrLd = 3,         // score row too short
  kErrTimeout = 4,    // bounded wait gave up
};

}  // namespace csa
