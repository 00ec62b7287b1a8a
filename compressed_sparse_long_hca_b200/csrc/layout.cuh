// Arena layout of the CSA / HCA cache, shared by the host code and the kernels.
//
// The split into a per-request state cache and a paged classic cache follows
// page "V4终于终于终于终于是来了", section "HCA——重度压缩注意力" (cache
// paragraph): the state cache holds, per request, the latest 128 raw tokens'
// KV and the tails that have not yet filled a 4- or 128-token window; the
// classic cache holds compressed entries in blocks of lcm(4, 128) = 128 raw
// tokens, i.e. 32 CSA entries and 1 HCA entry per block and layer.
//
// Arena (one caller-owned device buffer, every section 256-byte aligned):
//   header      error word (int32 code, int32 detail, int64 info)
//   lengths     int64 [n_layers][max_req]         tokens appended so far
//   capacity    int32 [max_req]                   blocks held by the request
//   block table int32 [max_req][max_blocks_per_req]  logical -> pool block
//   b_pos       fp32 [n_csa][8][D], [n_csa][8][d_I], [n_hca][128][D]
//   state       per request, per layer:
//                 window ring: fp8 [128][D-R] | bf16 [128][R] | fp32 [128]
//                 CSA tail:    fp32 c[8][D] | z[8][D] | ci[8][d_I] | zi[8][d_I]
//                 HCA tail:    fp32 c[128][D] | z[128][D]
//   pool        pool_blocks x block, block = per CSA layer
//                 fp8 [32][D-R] | bf16 [32][R] | fp32 scale [32] |
//                 index codes (32 keys x d_I/2 bytes, see below) | e8m0 [32][d_I/32]
//               then per HCA layer one row fp8 [D-R] | bf16 [R] | fp32 scale.
//
// Index-key codes inside a block are stored in the K-major "core matrix"
// order that tcgen05 reads without a swizzle: key s, 16-byte chunk c (32 E2M1
// values) lives at (s/8)*(CH*128) + c*128 + (s%8)*16, CH = d_I/32.  Four
// consecutive blocks therefore form one 128-key operand tile with a fixed
// 128-byte leading-dimension and CH*128-byte stride-dimension offset.
#pragma once
#include <stddef.h>
#include <stdint.h>

namespace csa {

constexpr int kWindow = 128;      // raw-token window
constexpr int kCsaM = 4;          // CSA compression ratio
constexpr int kCsaWin = 8;        // CSA window (2m, overlapping)
constexpr int kHcaM = 128;        // HCA compression ratio
constexpr int kBlockTokens = 128; // classic-cache block, lcm(4, 128)
constexpr int kCsaPerBlock = 32;

constexpr int64_t kAlign = 256;
__host__ __device__ constexpr int64_t align_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

struct Layout {
  // shapes
  int H, D, R, HI, dI;
  int n_csa, n_hca, n_layers;
  int max_req, max_blocks_per_req, pool_blocks;
  float rope_base;
  // arena base
  char* base;
  // section offsets from base
  int64_t off_err, off_len, off_cap, off_bt, off_bkv, off_bidx, off_bhca, off_state, off_pool;
  // row sections
  int64_t kv_fp8_bytes;     // D - R
  int64_t kv_bf16_bytes;    // 2R
  // state sizes
  int64_t ring_fp8, ring_bf16, ring_scale, ring_bytes;          // offsets inside a ring
  int64_t csa_tail_bytes, hca_tail_bytes;
  int64_t state_csa_layer, state_hca_layer, state_req;          // strides
  // block sizes
  int64_t blk_kv_bf16, blk_kv_scale, blk_idx_codes, blk_idx_scale, blk_csa_bytes;
  int64_t blk_hca_bf16, blk_hca_scale, blk_hca_bytes;
  int64_t block_bytes;
  int64_t total_bytes;

  __host__ __device__ int64_t* lengths() const { return reinterpret_cast<int64_t*>(base + off_len); }
  __host__ __device__ int32_t* capacity() const { return reinterpret_cast<int32_t*>(base + off_cap); }
  __host__ __device__ int32_t* block_table(int req) const {
    return reinterpret_cast<int32_t*>(base + off_bt) + (int64_t)req * max_blocks_per_req;
  }
  __host__ __device__ int32_t* err() const { return reinterpret_cast<int32_t*>(base + off_err); }
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
  // section of pool block `blk` that belongs to `layer`
  __host__ __device__ char* block(int64_t blk, int layer) const {
    int64_t o = off_pool + blk * block_bytes;
    if (layer < n_csa) o += (int64_t)layer * blk_csa_bytes;
    else o += (int64_t)n_csa * blk_csa_bytes + (int64_t)(layer - n_csa) * blk_hca_bytes;
    return base + o;
  }
};

// Device error word: first error wins.
enum DevErr : int32_t {
  kErrNone = 0,
  kErrBounds = 1,     // request id / block / index out of range
  kErrCapacity = 2,   // append beyond the request's blocks
  kErrLd = 3,         // score row too short
  kErrTimeout = 4,    // bounded wait gave up
};

}  // namespace csa
