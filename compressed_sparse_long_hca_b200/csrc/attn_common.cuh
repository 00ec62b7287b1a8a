// Pieces of the decode attention shared by the tensor-core kernel (the
// mixed FP8 / BF16 storage format) and the CUDA-core kernel (the fp32
// storage format): arguments, the rows of a query, and the fold of per-tile
// partials.
//
// Page "V4终于终于终于终于是来了", sections "CSA——压缩稀疏注意力" and
// "HCA——重度压缩注意力": a query attends to its selected (CSA) or all (HCA)
// compressed entries, then the 128 latest raw tokens; each head's sink logit
// enters the softmax denominator.  The rows are cut into tiles of 128; each
// tile gives (m_t, l_t, O_t).  The tiles are grouped into chunks of C
// consecutive tiles: the tiles of a chunk are folded in order into the
// chunk's (m_c, l_c, O_c), then the chunks are folded in order, the sink
// last.  C follows from the layer kind and the query's own tile count
// (attn_chunk_tiles), never from the batch.  Both storage formats and both launch variants use the fold below,
// so that the order and the rounding of the reduction depend on the query
// alone.
#pragma once
#include "common.cuh"

namespace csa {

constexpr int kTileRows = 128;
constexpr int kFoldBatch = 9;      // partials loaded at once by the fold kernel (a top-1024 query's 9 tiles)

// Tiles per chunk of the reduction: 1 on CSA layers (a top-k query has a
// handful of tiles, each a unit of parallel work); on HCA layers
// max(1, n_tiles / 8) for the query's own tile count, so that a short query
// keeps one tile per chunk (its tiles run in parallel) and a long one folds
// runs of tiles on chip (a query at 1M tokens: 65 tiles, 9 chunks of 8).  A
// chunk of one tile is that tile's partial exactly (folding into an empty
// result scales by e^0 = 1).
constexpr int kHcaChunkDiv = 8;
__host__ __device__ inline int attn_chunk_tiles(bool csa, int n_tiles) {
  return csa ? 1 : (n_tiles / kHcaChunkDiv > 1 ? n_tiles / kHcaChunkDiv : 1);
}

struct AttnArgs {
  Layout L;
  int layer;
  int n;
  const int32_t* req_ids;
  const void* q;       // BF16 (mixed format) or fp32 (fp32 format) [n][H][D]
  const int32_t* topk;
  int k;
  const float* sink;
  float scale;
  void* out;           // BF16 or fp32 [n][H][D], as q
  int G;              // heads per CTA (MMA N), 16 or 32
  // split launch only: partials of (query i, chunk c, head h)
  float* ws_o;        // [n][chunks_max][H][D]
  float2* ws_ml;      // [n][chunks_max][H]   (m_c, l_c); m_c = -inf: empty chunk
  int chunks_max;
  int f32;            // fp32 storage format: fp32 q and out
  // The lengths, window rows, q and sink are final before the previous grid
  // on the stream ends (that grid writes none of them): they may be read
  // before griddepcontrol.wait.  Top-k lists and compressed entries never are.
  int state_ready;
  // Chunk queries (q_per_req = C > 0, see visible_tokens): the C latest
  // tokens of each request were appended together, which overwrote the ring
  // rows of the C oldest window positions.  win_snap holds, per request of
  // the chunk (query i: request slot i / C), a copy of its ring taken before
  // that append; window positions below len - 128 are read from the copy.
  int q_per_req;
  const char* win_snap;
  // split launch only: the CTAs of one (query, head group) form a cluster
  // (one CTA per chunk) and fold the chunks' partials through distributed
  // shared memory instead of the workspace and attn_fold_kernel
  int cluster_fold;
};

struct QueryGeom {
  int req;
  bool csa;
  int64_t len;        // tokens of the request (the chunk included)
  const char* snap;   // chunk queries: the request's ring before the chunk's append
  int64_t t;          // query position
  int64_t n_entries, w0, n_win, n_list, total;
  int n_tiles;
  int chunk;          // tiles per chunk
  int n_chunks;
};

__device__ __forceinline__ bool query_geom(const AttnArgs& a, int i, QueryGeom& g, bool report) {
  const Layout& L = a.L;
  g.req = a.req_ids[i];
  if (g.req < 0 || g.req >= L.max_req) {
    if (report) set_err(L, kErrBounds, i);
    return false;
  }
  g.csa = a.layer < L.n_csa;
  g.len = L.lengths()[(int64_t)a.layer * L.max_req + g.req];
  const int64_t T = visible_tokens(g.len, a.q_per_req, i);
  if (T <= 0) {
    if (report) set_err(L, kErrBounds, 1000000 + i);
    return false;
  }
  g.snap = (a.q_per_req > 0 && a.win_snap != nullptr) ? a.win_snap + (int64_t)(i / a.q_per_req) * L.ring_bytes
                                                      : nullptr;
  g.t = T - 1;
  g.n_entries = g.csa ? T / kCsaM : T / kHcaM;
  g.w0 = g.t - (kWindow - 1) > 0 ? g.t - (kWindow - 1) : 0;
  g.n_win = g.t - g.w0 + 1;
  g.n_list = g.csa ? a.k : g.n_entries;
  g.total = g.n_list + g.n_win;
  g.n_tiles = (int)((g.total + kTileRows - 1) / kTileRows);
  g.chunk = attn_chunk_tiles(g.csa, g.n_tiles);
  g.n_chunks = (g.n_tiles + g.chunk - 1) / g.chunk;
  return true;
}

// Base of the window ring that holds position p (a window position of the
// query): the request's ring, or for a chunk query a position the chunk's
// own append has overwritten there, the copy taken before it.  The ring
// keeps positions len - 128 .. len - 1; the copy keeps the 128 positions
// before the chunk, which cover the rest of every window of a chunk of at
// most 128 queries.
__device__ __forceinline__ const char* ring_base(const AttnArgs& a, const QueryGeom& g, int64_t p) {
  return (g.snap != nullptr && p < g.len - kWindow) ? g.snap : a.L.state(g.req, a.layer);
}

// The fold of one partial into a running (m, l, O); shared by both launch
// variants so that they round identically.
__device__ __forceinline__ void fold_coef(float m, float mt, float& mn, float& al, float& be) {
  mn = fmaxf(m, mt);
  al = (m == -INFINITY) ? 0.f : expf(m - mn);
  be = expf(mt - mn);
}
__device__ __forceinline__ float fold_val(float o, float al, float ot, float be) {
  const float b = __fmul_rn(ot, be);
  return al == 0.f ? b : __fmaf_rn(o, al, b);
}
__device__ __forceinline__ void finish_coef(float m, float sk, float l, float& cm, float& den) {
  const float mu = fmaxf(m, sk);
  cm = expf(m - mu);
  den = __fmaf_rn(l, cm, expf(sk - mu));
}
__device__ __forceinline__ float finish_f32(float o, float cm, float den) {
  return __fdiv_rn(__fmul_rn(o, cm), den);
}
__device__ __forceinline__ uint16_t finish_val(float o, float cm, float den) {
  return bf16_rn(finish_f32(o, cm, den));
}

int attn_tiles_max(const Layout& L, int layer, int k);
int attn_chunks_max(const Layout& L, int layer, int k);
cudaError_t launch_attn_fold(const AttnArgs& a, cudaStream_t st);

}  // namespace csa
