// Host side of the C ABI declared in include/csa.h: configuration checks,
// arena layout, the host-side page allocator, launches and test helpers.
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <string>
#include <vector>

#include "csa.h"
#include "gemm_out.cuh"
#include "layout.cuh"

namespace csa {
cudaError_t launch_append(const Layout& L, int layer, int n, const int32_t* req_ids, int n_tok,
                          const float* c, const float* z, const float* ci, const float* zi,
                          cudaStream_t st);
cudaError_t launch_index_tc(const Layout& L, int layer, int n, const int32_t* req_ids, const float* q_idx,
                            const float* w, float* scores, int64_t ld, int32_t* n_valid, int ctas,
                            cudaStream_t st, int q_per_req = 0);
int topk_cluster_one_wave(int64_t ld, int n);
cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* n_valid, int n, int k,
                        int32_t* out, int32_t* err, int cluster, cudaStream_t st);
cudaError_t launch_attn_tc(const Layout& L, int layer, int n, const int32_t* req_ids, const uint16_t* q,
                           const int32_t* topk, int k, const float* sink, float scale, uint16_t* out, int G,
                           void* ws, cudaStream_t st, bool state_ready = false, int q_per_req = 0,
                           const char* win_snap = nullptr);
size_t attn_workspace_bytes(const Layout& L, int layer, int n, int k);
size_t attn_noalloc_scratch_bytes();
cudaError_t attn_noalloc_scratch(void** out);
cudaError_t launch_wait_probe(const Layout& L, uint64_t limit_ns, cudaStream_t st);
size_t index_topk_workspace_bytes(int n, int64_t ld);
cudaError_t launch_index_topk(const Layout& L, int layer, int n, const int32_t* req_ids, const float* q_idx,
                              const float* w, float* scores, int64_t ld, int32_t* n_valid, int k, int32_t* idx_out,
                              void* ws, int ctas, cudaStream_t st);
cudaError_t launch_index_f32(const Layout& L, int layer, int n, const int32_t* req_ids, const float* q_idx,
                             const float* w, float* scores, int64_t ld, int32_t* n_valid, int ctas_per_query,
                             cudaStream_t st, int q_per_req = 0);
cudaError_t launch_attn_f32(const Layout& L, int layer, int n, const int32_t* req_ids, const float* q,
                            const int32_t* topk, int k, const float* sink, float scale, float* out, void* ws,
                            cudaStream_t st, int q_per_req = 0, const char* win_snap = nullptr);
cudaError_t launch_chunk_prep(const Layout& L, int layer, int n, const int32_t* req_ids, int n_tok, int32_t* req_exp,
                              char* snap, cudaStream_t st);
cudaError_t launch_copy16(const void* src, void* dst, size_t bytes, cudaStream_t st);
int gemm_row_tiles(int n_out);
int gemm_k_tiles(int k_in, int groups);
size_t gemm_weight_bytes(int n_out, int k_in, int groups);
int gemm_max_tokens();
size_t gemm_workspace_bytes(int n_out, int k_in, int groups, int n_tok, int sms);
void gemm_pack_weight_host(const uint16_t* w, int n_out, int k_in, int groups, uint8_t* dst);
cudaError_t launch_gemm_bf16(const void* w_packed, int n_out, int k_in, int groups, const uint16_t* x, int n_tok,
                             const GemmOut& out, void* ws, int sms, cudaStream_t st);
cudaError_t gemm_read_error(int32_t* code, int32_t* detail, cudaStream_t st);
}  // namespace csa

namespace {
std::atomic<uint64_t> g_launches{0};
}

void csa::note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

using csa::Layout;

struct csa_cache {
  csa_cfg cfg;
  Layout L;
  std::vector<int32_t> free_pages;                // pool pages not held by a request
  std::vector<std::vector<int32_t>> req_pages;    // pages held by each request
  // csa_decode_step: the query's copy runs on a second stream (fork / join events)
  cudaStream_t side = nullptr;
  cudaEvent_t ev_fork = nullptr, ev_q = nullptr;
  ~csa_cache() {
    if (ev_q) cudaEventDestroy(ev_q);
    if (ev_fork) cudaEventDestroy(ev_fork);
    if (side) cudaStreamDestroy(side);
  }
};

namespace {

thread_local std::string g_err;

csa_status fail(csa_status s, const std::string& msg) {
  g_err = msg;
  return s;
}

csa_status cuda_fail(cudaError_t e, const char* what) {
  return fail(CSA_ERR_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

bool cfg_ok(const csa_cfg* c, std::string* why) {
  auto bad = [&](const char* m) { if (why) *why = m; return false; };
  if (!c) return bad("cfg is NULL");
  if (c->n_csa_layers < 0 || c->n_hca_layers < 0 || c->n_csa_layers + c->n_hca_layers < 1)
    return bad("need at least one layer");
  if (c->H < 1 || c->H > 128) return bad("H must be in [1, 128]");
  if (c->D < 64 || c->D > 512 || c->D % 32) return bad("D must be a multiple of 32 in [64, 512]");
  if (c->D_rope < 16 || c->D_rope > 64 || c->D_rope % 2 || c->D_rope >= c->D || (c->D - c->D_rope) % 16)
    return bad("D_rope must be even, in [16, 64], < D, with D - D_rope a multiple of 16");
  if (c->n_csa_layers > 0) {
    if (c->H_I < 1 || c->H_I > 64) return bad("H_I must be in [1, 64]");
    if (c->d_I < 32 || c->d_I > 128 || c->d_I % 32) return bad("d_I must be 32, 64, 96 or 128");
  }
  if (c->window != csa::kWindow) return bad("window must be 128");
  if (c->max_requests < 1) return bad("max_requests must be >= 1");
  if (c->max_pages_per_request < 1) return bad("max_pages_per_request must be >= 1");
  if (c->pool_pages < 1) return bad("pool_pages must be >= 1");
  if (!(c->rope_base > 1.f)) return bad("rope_base must be > 1");
  if (c->fmt != CSA_FMT_MIXED && c->fmt != CSA_FMT_F32) return bad("fmt must be CSA_FMT_MIXED or CSA_FMT_F32");
  return true;
}

Layout make_layout(const csa_cfg& c) {
  using csa::align_up;
  const int64_t A = csa::kAlign;
  Layout L{};
  L.H = c.H; L.D = c.D; L.R = c.D_rope;
  L.HI = c.n_csa_layers ? c.H_I : 0;
  L.dI = c.n_csa_layers ? c.d_I : 32;
  L.n_csa = c.n_csa_layers; L.n_hca = c.n_hca_layers; L.n_layers = c.n_csa_layers + c.n_hca_layers;
  L.max_req = c.max_requests; L.max_pages_per_req = c.max_pages_per_request;
  L.pool_pages = c.pool_pages; L.rope_base = c.rope_base;
  L.fmt = c.fmt;
  const bool f32 = c.fmt == CSA_FMT_F32;
  L.kv_fp8_bytes = c.D - c.D_rope;
  L.kv_bf16_bytes = 2 * (int64_t)c.D_rope;
  // window ring
  L.ring_fp8 = 0;
  L.ring_bf16 = align_up(csa::kWindow * L.kv_fp8_bytes, 128);
  L.ring_scale = L.ring_bf16 + align_up(csa::kWindow * L.kv_bf16_bytes, 128);
  L.ring_bytes = L.ring_scale + align_up(csa::kWindow * 4, 128);
  if (f32) L.ring_bytes = align_up((int64_t)csa::kWindow * c.D * 4, 128);
  L.csa_tail_bytes = align_up((int64_t)csa::kCsaWin * (2 * c.D + 2 * L.dI) * 4, 128);
  L.hca_tail_bytes = align_up((int64_t)csa::kHcaM * 2 * c.D * 4, 128);
  L.state_csa_layer = L.ring_bytes + L.csa_tail_bytes;
  L.state_hca_layer = L.ring_bytes + L.hca_tail_bytes;
  L.state_req = align_up(L.n_csa * L.state_csa_layer + L.n_hca * L.state_hca_layer, A);
  // classic-cache page sections (a page = 4 blocks = 512 raw tokens)
  L.CHs = (L.dI / 32 + 1) / 2 * 2;
  const int64_t P = csa::kCsaPerPage, PH = csa::kHcaPerPage;
  L.pg_csa_bf16 = align_up(P * L.kv_fp8_bytes, 128);
  L.pg_csa_scale = L.pg_csa_bf16 + align_up(P * L.kv_bf16_bytes, 128);
  L.pg_idx_codes = L.pg_csa_scale + align_up(P * 4, 128);
  L.pg_idx_sf = L.pg_idx_codes + P * L.CHs * 16;          // codes and scales are adjacent
  L.idx_tile_bytes = P * L.CHs * 16 + csa::kSfChunk;
  L.pg_csa_bytes = align_up(L.pg_idx_codes + L.idx_tile_bytes, 128);
  L.pg_hca_bf16 = align_up(PH * L.kv_fp8_bytes, 16);
  L.pg_hca_scale = L.pg_hca_bf16 + align_up(PH * L.kv_bf16_bytes, 16);
  L.pg_hca_bytes = align_up(L.pg_hca_scale + PH * 4, 128);
  L.pg_idx_f32 = 0;
  if (f32) {   // fp32 rows [P][D], then (CSA) fp32 keys [P][d_I]
    L.pg_idx_f32 = align_up(P * c.D * 4, 128);
    L.pg_csa_bytes = align_up(L.pg_idx_f32 + P * L.dI * 4, 128);
    L.pg_hca_bytes = align_up(PH * c.D * 4, 128);
  }
  L.page_bytes = align_up(L.n_csa * L.pg_csa_bytes + L.n_hca * L.pg_hca_bytes, A);
  // arena sections
  int64_t o = 0;
  L.off_err = o; o += A;
  L.off_tick = o; o = align_up(o + (int64_t)L.n_layers * L.max_req * 4, A);
  L.off_len = o; o = align_up(o + (int64_t)L.n_layers * L.max_req * 8, A);
  L.off_cap = o; o = align_up(o + (int64_t)L.max_req * 4, A);
  L.off_pt = o; o = align_up(o + (int64_t)L.max_req * L.max_pages_per_req * 4, A);
  L.off_theta = o; o = align_up(o + (int64_t)(L.R / 2) * 8, A);
  L.off_bkv = o; o = align_up(o + (int64_t)L.n_csa * csa::kCsaWin * c.D * 4, A);
  L.off_bidx = o; o = align_up(o + (int64_t)L.n_csa * csa::kCsaWin * L.dI * 4, A);
  L.off_bhca = o; o = align_up(o + (int64_t)L.n_hca * csa::kHcaM * c.D * 4, A);
  L.off_state = o; o = align_up(o + (int64_t)L.max_req * L.state_req, A);
  L.off_pool = o; o = align_up(o + (int64_t)L.pool_pages * L.page_bytes, A);
  L.total_bytes = o;
  L.base = nullptr;
  return L;
}

int sm_count() {
  int dev = 0, v = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return v;
}

bool layer_ok(const csa_cache* c, int32_t layer) { return c && layer >= 0 && layer < c->L.n_layers; }

}  // namespace

extern "C" {

size_t csa_cache_required_bytes(const csa_cfg* cfg) {
  if (!cfg_ok(cfg, nullptr)) return 0;
  return (size_t)make_layout(*cfg).total_bytes;
}

csa_status csa_cache_init(const csa_cfg* cfg, void* dev_mem, size_t bytes, const float* b_pos_csa,
                          const float* b_pos_idx, const float* b_pos_hca, csa_cache_t** out) {
  std::string why;
  if (!out) return fail(CSA_ERR_ARG, "out is NULL");
  *out = nullptr;
  if (!cfg_ok(cfg, &why)) return fail(CSA_ERR_ARG, why);
  if (!dev_mem || (reinterpret_cast<uintptr_t>(dev_mem) % csa::kAlign))
    return fail(CSA_ERR_ARG, "dev_mem must be a 256-byte aligned device pointer");
  Layout L = make_layout(*cfg);
  if ((int64_t)bytes < L.total_bytes) return fail(CSA_ERR_CAPACITY, "arena smaller than required bytes");
  if (cfg->n_csa_layers > 0 && (!b_pos_csa || !b_pos_idx)) return fail(CSA_ERR_ARG, "CSA position biases missing");
  if (cfg->n_hca_layers > 0 && !b_pos_hca) return fail(CSA_ERR_ARG, "HCA position biases missing");
  L.base = static_cast<char*>(dev_mem);
  cudaError_t e = cudaMemset(L.base, 0, (size_t)L.off_bkv);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(arena header)");
  if (L.n_csa) {
    e = cudaMemcpy(L.base + L.off_bkv, b_pos_csa, (size_t)L.n_csa * csa::kCsaWin * L.D * 4, cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
      e = cudaMemcpy(L.base + L.off_bidx, b_pos_idx, (size_t)L.n_csa * csa::kCsaWin * L.dI * 4, cudaMemcpyHostToDevice);
  }
  if (e == cudaSuccess && L.n_hca)
    e = cudaMemcpy(L.base + L.off_bhca, b_pos_hca, (size_t)L.n_hca * csa::kHcaM * L.D * 4, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(position biases)");
  {
    std::vector<double> th(L.R / 2);
    for (int i = 0; i < L.R / 2; ++i) th[i] = std::pow((double)cfg->rope_base, -2.0 * i / (double)L.R);
    e = cudaMemcpy(L.base + L.off_theta, th.data(), th.size() * 8, cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(rope frequencies)");
  }
  csa_cache* c = new (std::nothrow) csa_cache();
  if (!c) return fail(CSA_ERR_CAPACITY, "host allocation failed");
  c->cfg = *cfg;
  c->L = L;
  c->req_pages.assign(cfg->max_requests, {});
  if ((e = cudaStreamCreateWithFlags(&c->side, cudaStreamNonBlocking)) != cudaSuccess ||
      (e = cudaEventCreateWithFlags(&c->ev_fork, cudaEventDisableTiming)) != cudaSuccess ||
      (e = cudaEventCreateWithFlags(&c->ev_q, cudaEventDisableTiming)) != cudaSuccess) {
    delete c;
    return cuda_fail(e, "stream / event creation");
  }
  // Hand pool pages out in a fixed pseudo-random order, so that a request's
  // pages are scattered through the pool and every access goes through the
  // page table.
  c->free_pages.resize(cfg->pool_pages);
  for (int32_t b = 0; b < cfg->pool_pages; ++b) c->free_pages[b] = b;
  uint64_t s = 0x9E3779B97F4A7C15ull;
  for (int32_t b = cfg->pool_pages - 1; b > 0; --b) {
    s ^= s << 13; s ^= s >> 7; s ^= s << 17;
    std::swap(c->free_pages[b], c->free_pages[s % (uint64_t)(b + 1)]);
  }
  *out = c;
  return CSA_OK;
}

void csa_cache_destroy(csa_cache_t* cache) { delete cache; }

static csa_status reset_lengths(csa_cache* c, int32_t req) {
  const Layout& L = c->L;
  for (int l = 0; l < L.n_layers; ++l) {
    cudaError_t e = cudaMemset(L.lengths() + (int64_t)l * L.max_req + req, 0, 8);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(length)");
  }
  return CSA_OK;
}

csa_status csa_request_free(csa_cache_t* c, int32_t req) {
  if (!c || req < 0 || req >= c->L.max_req) return fail(CSA_ERR_ARG, "bad request id");
  auto& held = c->req_pages[req];
  c->free_pages.insert(c->free_pages.end(), held.rbegin(), held.rend());
  held.clear();
  cudaError_t e = cudaMemset(c->L.capacity() + req, 0, 4);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(capacity)");
  return reset_lengths(c, req);
}

csa_status csa_request_alloc(csa_cache_t* c, int32_t req, int64_t capacity_tokens) {
  if (!c || req < 0 || req >= c->L.max_req) return fail(CSA_ERR_ARG, "bad request id");
  if (capacity_tokens < 1) return fail(CSA_ERR_ARG, "capacity_tokens must be >= 1");
  csa_status s = csa_request_free(c, req);
  if (s != CSA_OK) return s;
  const int64_t nb = (capacity_tokens + csa::kPageTokens - 1) / csa::kPageTokens;
  if (nb > c->L.max_pages_per_req) return fail(CSA_ERR_CAPACITY, "capacity exceeds max_pages_per_request");
  if (nb > (int64_t)c->free_pages.size()) return fail(CSA_ERR_CAPACITY, "page pool exhausted");
  auto& held = c->req_pages[req];
  held.assign(c->free_pages.end() - nb, c->free_pages.end());
  std::reverse(held.begin(), held.end());
  c->free_pages.resize(c->free_pages.size() - nb);
  cudaError_t e = cudaMemcpy(c->L.page_table(req), held.data(), nb * 4, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(page table)");
  const int32_t nb32 = (int32_t)nb;
  e = cudaMemcpy(c->L.capacity() + req, &nb32, 4, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(capacity)");
  return CSA_OK;
}

csa_status csa_compress_append(csa_cache_t* c, int32_t layer, int32_t n, const int32_t* req_ids,
                               int32_t n_tok, const float* kv_cand, const float* kv_gate,
                               const float* idx_cand, const float* idx_gate, csa_stream_t stream) {
  if (!layer_ok(c, layer)) return fail(CSA_ERR_ARG, "bad layer");
  if (n < 0 || n > 65535) return fail(CSA_ERR_ARG, "n must be in [0, 65535]");
  if (n == 0) return CSA_OK;
  if (n_tok < 1) return fail(CSA_ERR_ARG, "n_tok must be >= 1");
  if (!req_ids || !kv_cand || !kv_gate) return fail(CSA_ERR_ARG, "NULL input");
  const bool is_csa = layer < c->L.n_csa;
  if (is_csa && (!idx_cand || !idx_gate)) return fail(CSA_ERR_ARG, "CSA layer needs index-key inputs");
  cudaError_t e = csa::launch_append(c->L, layer, n, req_ids, n_tok, kv_cand, kv_gate,
                                     idx_cand, idx_gate, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "append launch");
  return CSA_OK;
}

// Chunk queries (csa_prefill_chunk): q_per_req queries per request for its
// latest tokens, and the copy of each request's ring taken before the
// chunk's append.  Zero for decode queries.
struct ChunkQ {
  int q_per_req;
  const char* snap;
};

static csa_status index_scores_impl(const csa_cache_t* c, int32_t layer, int32_t n, const int32_t* req_ids,
                                    const float* q_idx, const float* w, float* scores, int64_t ld,
                                    int32_t* n_valid, csa_variant variant, csa_stream_t stream, ChunkQ cq) {
  if (!layer_ok(c, layer) || layer >= c->L.n_csa) return fail(CSA_ERR_ARG, "index scores need a CSA layer");
  if (n < 0 || n > 65535) return fail(CSA_ERR_ARG, "n must be in [0, 65535]");
  if (n == 0) return CSA_OK;
  if (!req_ids || !q_idx || !w || !scores || !n_valid) return fail(CSA_ERR_ARG, "NULL argument");
  if (ld < 1) return fail(CSA_ERR_ARG, "ld must be >= 1");
  if (variant < CSA_VARIANT_AUTO || variant > CSA_VARIANT_LOW_OCC) return fail(CSA_ERR_ARG, "bad variant");
  const int sms = sm_count();
  if (sms <= 0) return fail(CSA_ERR_CUDA, "cannot query the SM count");
  cudaError_t e;
  if (c->L.fmt == csa::kFmtF32) {
    // fp32 keys on the CUDA cores: one thread per key; the variants only
    // change how many CTAs share a query (the per-key arithmetic is fixed)
    const bool low = variant == CSA_VARIANT_LOW_OCC || (variant == CSA_VARIANT_AUTO && n < sms);
    const int per_q = low ? std::max(1, (4 * sms + n - 1) / n) : 1;
    e = csa::launch_index_f32(c->L, layer, n, req_ids, q_idx, w, scores, ld, n_valid, std::min(per_q, 1024),
                              (cudaStream_t)stream, cq.q_per_req);
  } else {
    // Persistent CTAs over the flattened (query, tile) list: two per SM (AUTO,
    // HIGH_OCC: their tcgen05 issue latencies overlap), or one per SM
    // (LOW_OCC).  The CTAs own different tile ranges in the two grids; a
    // key's score does not depend on which CTA computes it.
    const int ctas = variant == CSA_VARIANT_LOW_OCC ? sms : 2 * sms;
    e = csa::launch_index_tc(c->L, layer, n, req_ids, q_idx, w, scores, ld, n_valid, ctas,
                             (cudaStream_t)stream, cq.q_per_req);
  }
  if (e != cudaSuccess) return cuda_fail(e, "index launch");
  return CSA_OK;
}

csa_status csa_index_scores(const csa_cache_t* c, int32_t layer, int32_t n, const int32_t* req_ids,
                            const float* q_idx, const float* w, float* scores, int64_t ld,
                            int32_t* n_valid, csa_variant variant, csa_stream_t stream) {
  return index_scores_impl(c, layer, n, req_ids, q_idx, w, scores, ld, n_valid, variant, stream, ChunkQ{0, nullptr});
}

csa_status csa_topk(const float* scores, int64_t ld, const int32_t* n_valid, int32_t n, int32_t k,
                    int32_t* idx_out, csa_variant variant, csa_stream_t stream) {
  if (n < 0 || n > 65535) return fail(CSA_ERR_ARG, "n must be in [0, 65535]");
  if (n == 0) return CSA_OK;
  if (!scores || !n_valid || !idx_out) return fail(CSA_ERR_ARG, "NULL argument");
  if (k < 1 || ld < 1) return fail(CSA_ERR_ARG, "k and ld must be >= 1");
  if (variant < CSA_VARIANT_AUTO || variant > CSA_VARIANT_LOW_OCC) return fail(CSA_ERR_ARG, "bad variant");
  // One thread-block cluster per query: 16 CTAs for LOW_OCC (8 where the
  // device cannot co-schedule 16), 8 for HIGH_OCC; AUTO takes the largest
  // of 16, 8 and 4 whose n clusters the device holds at once (one CTA of
  // 1024 threads per SM: 32 queries take clusters of 4 rather than two
  // waves of 8).  A row of at most 4096 scores fits one thread block: AUTO
  // and HIGH_OCC then select it in a single block (no cluster round trips),
  // LOW_OCC in a cluster of 8.  The selection is exact, so every form
  // returns identical indices.
  int cluster = 8;
  if (ld <= 4096) cluster = variant == CSA_VARIANT_LOW_OCC ? 8 : 1;
  else if (variant == CSA_VARIANT_LOW_OCC) cluster = 16;
  else if (variant == CSA_VARIANT_AUTO) cluster = csa::topk_cluster_one_wave(ld, n);
  cudaError_t e = csa::launch_topk(scores, ld, n_valid, n, k, idx_out, nullptr, cluster, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "topk launch");
  return CSA_OK;
}

size_t csa_index_topk_workspace_bytes(const csa_cache_t* c, int32_t n, int64_t ld) {
  if (!c || n < 1 || n > 65535 || ld < 1) return 0;
  if (c->L.fmt == csa::kFmtF32) return 16;   // the fp32 format runs the two separate kernels
  return csa::index_topk_workspace_bytes(n, ld);
}

csa_status csa_index_topk(const csa_cache_t* c, int32_t layer, int32_t n, const int32_t* req_ids,
                          const float* q_idx, const float* w, float* scores, int64_t ld, int32_t* n_valid,
                          int32_t k, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                          csa_variant variant, csa_stream_t stream) {
  if (!layer_ok(c, layer) || layer >= c->L.n_csa) return fail(CSA_ERR_ARG, "index scores need a CSA layer");
  if (n < 0 || n > 65535) return fail(CSA_ERR_ARG, "n must be in [0, 65535]");
  if (n == 0) return CSA_OK;
  if (!req_ids || !q_idx || !w || !scores || !n_valid || !idx_out) return fail(CSA_ERR_ARG, "NULL argument");
  if (ld < 1 || k < 1) return fail(CSA_ERR_ARG, "k and ld must be >= 1");
  if (variant < CSA_VARIANT_AUTO || variant > CSA_VARIANT_LOW_OCC) return fail(CSA_ERR_ARG, "bad variant");
  if (c->L.fmt == csa::kFmtF32) {   // fp32 keys: the CUDA-core indexer, then the top-k kernel
    csa_status st = csa_index_scores(c, layer, n, req_ids, q_idx, w, scores, ld, n_valid, variant, stream);
    if (st != CSA_OK) return st;
    return csa_topk(scores, ld, n_valid, n, k, idx_out, variant, stream);
  }
  const size_t need = csa::index_topk_workspace_bytes(n, ld);
  if (!workspace || workspace_bytes < need || reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(CSA_ERR_ARG, "workspace must be 256-byte aligned and hold csa_index_topk_workspace_bytes");
  const int sms = sm_count();
  if (sms <= 0) return fail(CSA_ERR_CUDA, "cannot query the SM count");
  // the same persistent grid for either variant (the selection is exact)
  cudaError_t e = csa::launch_index_topk(c->L, layer, n, req_ids, q_idx, w, scores, ld, n_valid, k, idx_out,
                                         workspace, 2 * sms, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "fused index + top-k launch");
  return CSA_OK;
}

size_t csa_attn_workspace_bytes(const csa_cache_t* c, int32_t layer, int32_t n, int32_t k) {
  if (!layer_ok(c, layer) || n < 0 || n > 65535) return 0;
  const bool is_csa = layer < c->L.n_csa;
  if (is_csa && (k < 1 || k > 8192)) return 0;
  return csa::attn_workspace_bytes(c->L, layer, n, is_csa ? k : 0);
}

// Whether a launch of n queries takes the split attention (with a workspace).
static bool attn_split(const Layout& L, int32_t n, csa_variant variant, bool ws_ok) {
  const int G = L.H <= 16 ? 16 : 32;
  const int ctas = n * ((L.H + G - 1) / G);
  return variant == CSA_VARIANT_LOW_OCC || (variant == CSA_VARIANT_AUTO && ws_ok && ctas < sm_count());
}

static csa_status decode_attn_impl(const csa_cache_t* c, int32_t layer, int32_t n, const int32_t* req_ids,
                                   const void* q, const int32_t* topk_idx, int32_t k, const float* sink,
                                   float scale, void* out, void* workspace, size_t workspace_bytes,
                                   csa_variant variant_flags, csa_stream_t stream, ChunkQ cq) {
  const int flags = (int)variant_flags & ~0xFF;
  const csa_variant variant = (csa_variant)((int)variant_flags & 0xFF);
  if (flags & ~CSA_ATTN_STATE_READY) return fail(CSA_ERR_ARG, "unknown variant flag");
  if (!layer_ok(c, layer)) return fail(CSA_ERR_ARG, "bad layer");
  if (n < 0 || n > 65535) return fail(CSA_ERR_ARG, "n must be in [0, 65535]");
  if (n == 0) return CSA_OK;
  if (!req_ids || !q || !sink || !out) return fail(CSA_ERR_ARG, "NULL argument");
  if (reinterpret_cast<uintptr_t>(q) % 16) return fail(CSA_ERR_ARG, "q must be 16-byte aligned");
  const bool is_csa = layer < c->L.n_csa;
  if (is_csa && (!topk_idx || k < 1)) return fail(CSA_ERR_ARG, "CSA layer needs topk_idx and k >= 1");
  if (!is_csa && topk_idx) return fail(CSA_ERR_ARG, "HCA layer takes topk_idx == NULL");
  if (!(scale > 0.f)) return fail(CSA_ERR_ARG, "scale must be > 0");
  if (variant < CSA_VARIANT_AUTO || variant > CSA_VARIANT_LOW_OCC) return fail(CSA_ERR_ARG, "bad variant");
  if (is_csa && k > 8192) return fail(CSA_ERR_ARG, "k must be <= 8192");
  const int kk = is_csa ? k : 0;
  const size_t need = csa::attn_workspace_bytes(c->L, layer, n, kk);
  const bool ws_ok = workspace != nullptr && workspace_bytes >= need &&
                     reinterpret_cast<uintptr_t>(workspace) % 16 == 0;
  if (variant == CSA_VARIANT_LOW_OCC && !ws_ok)
    return fail(CSA_ERR_ARG, "the split launch needs a 16-byte aligned workspace of csa_attn_workspace_bytes");
  // 32 heads per CTA (16 when H <= 16).  Whole-query launch when one CTA per
  // (query, head group) already covers the SMs, split launch otherwise.  Both
  // compute the same tiles and fold them in the same order.
  const int G = c->L.H <= 16 ? 16 : 32;
  const bool split = attn_split(c->L, n, variant, ws_ok);
  cudaError_t e =
      c->L.fmt == csa::kFmtF32
          ? csa::launch_attn_f32(c->L, layer, n, req_ids, static_cast<const float*>(q), topk_idx, kk, sink, scale,
                                 static_cast<float*>(out), split ? workspace : nullptr, (cudaStream_t)stream,
                                 cq.q_per_req, cq.snap)
          : csa::launch_attn_tc(c->L, layer, n, req_ids, static_cast<const uint16_t*>(q), topk_idx, kk, sink,
                                scale, static_cast<uint16_t*>(out), G, split ? workspace : nullptr,
                                (cudaStream_t)stream, (flags & CSA_ATTN_STATE_READY) != 0, cq.q_per_req, cq.snap);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return CSA_OK;
}

csa_status csa_hca_decode_attn(const csa_cache_t* c, int32_t layer, int32_t n, const int32_t* req_ids,
                               const void* q, const int32_t* topk_idx, int32_t k, const float* sink,
                               float scale, void* out, void* workspace, size_t workspace_bytes,
                               csa_variant variant_flags, csa_stream_t stream) {
  return decode_attn_impl(c, layer, n, req_ids, q, topk_idx, k, sink, scale, out, workspace, workspace_bytes,
                          variant_flags, stream, ChunkQ{0, nullptr});
}

csa_status csa_hca_decode_attn_noalloc(const csa_cache_t* c, int32_t layer, int32_t n,
                                       const int32_t* req_ids, const void* q, const int32_t* topk_idx,
                                       int32_t k, const float* sink, float scale, void* out,
                                       csa_stream_t stream) {
  if (!layer_ok(c, layer)) return fail(CSA_ERR_ARG, "bad layer");
  if (n < 0 || n > 65535) return fail(CSA_ERR_ARG, "n must be in [0, 65535]");
  if (n == 0) return CSA_OK;
  if (!req_ids || !q || !sink || !out) return fail(CSA_ERR_ARG, "NULL argument");
  if (reinterpret_cast<uintptr_t>(q) % 16) return fail(CSA_ERR_ARG, "q must be 16-byte aligned");
  const bool is_csa = layer < c->L.n_csa;
  if (is_csa && (!topk_idx || k < 1)) return fail(CSA_ERR_ARG, "CSA layer needs topk_idx and k >= 1");
  if (!is_csa && topk_idx) return fail(CSA_ERR_ARG, "HCA layer takes topk_idx == NULL");
  if (!(scale > 0.f)) return fail(CSA_ERR_ARG, "scale must be > 0");
  if (is_csa && k > 8192) return fail(CSA_ERR_ARG, "k must be <= 8192");
  const int kk = is_csa ? k : 0;
  const size_t need = csa::attn_workspace_bytes(c->L, layer, n, kk);
  if (need > csa::attn_noalloc_scratch_bytes())
    return fail(CSA_ERR_CAPACITY, "this batch needs " + std::to_string(need) +
                                      " bytes of scratch; the built-in array holds " +
                                      std::to_string(csa::attn_noalloc_scratch_bytes()) +
                                      " (use a smaller batch or csa_hca_decode_attn with a workspace)");
  void* ws = nullptr;
  cudaError_t e = csa::attn_noalloc_scratch(&ws);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(scratch)");
  const int G = c->L.H <= 16 ? 16 : 32;
  e = c->L.fmt == csa::kFmtF32
          ? csa::launch_attn_f32(c->L, layer, n, req_ids, static_cast<const float*>(q), topk_idx, kk, sink, scale,
                                 static_cast<float*>(out), ws, (cudaStream_t)stream)
          : csa::launch_attn_tc(c->L, layer, n, req_ids, static_cast<const uint16_t*>(q), topk_idx, kk, sink,
                                scale, static_cast<uint16_t*>(out), G, ws, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return CSA_OK;
}

uint64_t csa_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

csa_status csa_check_device_error(csa_cache_t* c, csa_stream_t stream) {
  if (!c) return fail(CSA_ERR_ARG, "cache is NULL");
  cudaError_t e = cudaStreamSynchronize((cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int32_t w[4] = {0, 0, 0, 0};
  e = cudaMemcpy(w, c->L.err(), 16, cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(error word)");
  if (w[0] == 0) return CSA_OK;
  const int32_t zero[4] = {0, 0, 0, 0};
  e = cudaMemcpy(c->L.err(), zero, 16, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(error word reset)");
  char msg[160];
  switch (w[0]) {
    case csa::kErrBounds:
      snprintf(msg, sizeof msg, "device: index out of range (detail %d; %d %d)", w[1], w[2], w[3]);
      return fail(CSA_ERR_DEVICE_BOUNDS, msg);
    case csa::kErrCapacity:
      snprintf(msg, sizeof msg, "device: append beyond the capacity of request %d", w[1]);
      return fail(CSA_ERR_CAPACITY, msg);
    case csa::kErrLd:
      snprintf(msg, sizeof msg, "device: score row too short for query %d", w[1]);
      return fail(CSA_ERR_DEVICE_BOUNDS, msg);
    case csa::kErrTimeout:
      snprintf(msg, sizeof msg, "device: bounded wait gave up (detail %d)", w[1]);
      return fail(CSA_ERR_DEVICE_TIMEOUT, msg);
    default:
      snprintf(msg, sizeof msg, "device: error %d (detail %d)", w[0], w[1]);
      return fail(CSA_ERR_DEVICE_BOUNDS, msg);
  }
}

const char* csa_last_error(void) { return g_err.c_str(); }

// ---- one decode step with host buffers

namespace {

// Byte layout of csa_decode_step's packed host input and of its device
// scratch (every field on a 256-byte boundary).
struct StepLayout {
  int64_t c, z, ci, zi, qi, w, q, q_bytes, in_bytes;            // host input (and its device copy)
  int64_t d_scores, d_nv, d_idx, d_ws, d_out, out_bytes, dev_bytes, ld;
  size_t ws_bytes;
};

// The device's address of page-locked (pinned or registered) host memory,
// or null for any other memory (pageable host memory, device memory).
const void* mapped_host(const void* p) {
  cudaPointerAttributes at{};
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    (void)cudaGetLastError();
    return nullptr;
  }
  return at.type == cudaMemoryTypeHost ? at.devicePointer : nullptr;
}

StepLayout step_layout(const csa_cache* c, int32_t layer, int32_t n, int32_t k) {
  const Layout& L = c->L;
  const bool csa = layer < L.n_csa;
  const int64_t qb = L.fmt == csa::kFmtF32 ? 4 : 2;
  auto al = [](int64_t x) { return (x + 255) / 256 * 256; };
  StepLayout s{};
  int64_t o = 0;
  s.c = o;  o += al((int64_t)n * L.D * 4);
  s.z = o;  o += al((int64_t)n * L.D * 4);
  if (csa) {
    s.ci = o; o += al((int64_t)n * L.dI * 4);
    s.zi = o; o += al((int64_t)n * L.dI * 4);
    s.qi = o; o += al((int64_t)n * L.HI * L.dI * 4);
    s.w = o;  o += al((int64_t)n * L.HI * 4);
  }
  s.q = o;
  s.q_bytes = (int64_t)n * L.H * L.D * qb;
  o += al(s.q_bytes);
  s.in_bytes = o;
  s.ld = csa ? std::max<int64_t>((int64_t)L.max_pages_per_req * csa::kCsaPerPage, 128) : 0;
  s.d_scores = o; o += al((int64_t)n * s.ld * 4);
  s.d_nv = o;     o += al((int64_t)n * 4);
  s.d_idx = o;    o += al((int64_t)n * (csa ? k : 0) * 4);
  s.ws_bytes = csa::attn_workspace_bytes(L, layer, n, csa ? k : 0);
  s.d_ws = o;     o += al((int64_t)s.ws_bytes);
  s.out_bytes = s.q_bytes;
  s.d_out = o;    o += al(s.out_bytes);
  s.dev_bytes = o;
  return s;
}

}  // namespace

size_t csa_decode_step_input_bytes(const csa_cache_t* c, int32_t layer, int32_t n) {
  if (!layer_ok(c, layer) || n < 1 || n > 65535) return 0;
  return (size_t)step_layout(c, layer, n, 1).in_bytes;
}

size_t csa_decode_step_dev_bytes(const csa_cache_t* c, int32_t layer, int32_t n, int32_t k) {
  if (!layer_ok(c, layer) || n < 1 || n > 65535) return 0;
  if (layer < c->L.n_csa && (k < 1 || k > 8192)) return 0;
  return (size_t)step_layout(c, layer, n, k).dev_bytes;
}

csa_status csa_decode_step(csa_cache_t* c, int32_t layer, int32_t n, const int32_t* req_ids, int32_t k,
                           const float* sink, float scale, const void* host_in, void* host_out, void* dev_buf,
                           size_t dev_bytes, csa_stream_t stream) {
  if (!layer_ok(c, layer)) return fail(CSA_ERR_ARG, "bad layer");
  if (n < 1 || n > 65535) return fail(CSA_ERR_ARG, "n must be in [1, 65535]");
  const bool csa = layer < c->L.n_csa;
  if (csa && (k < 1 || k > 8192)) return fail(CSA_ERR_ARG, "a CSA layer needs 1 <= k <= 8192");
  if (!req_ids || !sink || !host_in || !host_out || !dev_buf) return fail(CSA_ERR_ARG, "NULL argument");
  if (reinterpret_cast<uintptr_t>(dev_buf) % 256) return fail(CSA_ERR_ARG, "dev_buf must be 256-byte aligned");
  const StepLayout sl = step_layout(c, layer, n, csa ? k : 0);
  if (dev_bytes < (size_t)sl.dev_bytes) return fail(CSA_ERR_ARG, "dev_buf smaller than csa_decode_step_dev_bytes");
  char* d = static_cast<char*>(dev_buf);
  const char* h = static_cast<const char*>(host_in);
  cudaStream_t st = (cudaStream_t)stream;
  // Page-locked host buffers are read and written by the kernels over the
  // bus (a copy kernel for the small inputs, the attention's own output
  // stores): a copy-engine transfer costs about 12 us of fixed latency on the
  // step's critical path.  Other host memory goes through copies.
  const void* in_dev = mapped_host(host_in);
  void* out_dev = const_cast<void*>(mapped_host(host_out));
  // inputs before q (for the append and the selection) first; q, which only
  // the attention reads, on the cache's second stream beside them
  cudaError_t e = in_dev != nullptr ? csa::launch_copy16(in_dev, d, (size_t)sl.q, st)
                                    : cudaMemcpyAsync(d, h, (size_t)sl.q, cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess) e = cudaEventRecord(c->ev_fork, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(c->side, c->ev_fork, 0);
  if (e == cudaSuccess)
    e = in_dev != nullptr
            ? csa::launch_copy16(static_cast<const char*>(in_dev) + sl.q, d + sl.q, (size_t)sl.q_bytes, c->side)
            : cudaMemcpyAsync(d + sl.q, h + sl.q, (size_t)sl.q_bytes, cudaMemcpyHostToDevice, c->side);
  if (e == cudaSuccess) e = cudaEventRecord(c->ev_q, c->side);
  if (e != cudaSuccess) return cuda_fail(e, "decode step input copies");
  csa_status r = csa_compress_append(c, layer, n, req_ids, 1, reinterpret_cast<const float*>(d + sl.c),
                                     reinterpret_cast<const float*>(d + sl.z),
                                     csa ? reinterpret_cast<const float*>(d + sl.ci) : nullptr,
                                     csa ? reinterpret_cast<const float*>(d + sl.zi) : nullptr, stream);
  int32_t* idx = csa ? reinterpret_cast<int32_t*>(d + sl.d_idx) : nullptr;
  if (r == CSA_OK && csa) {
    float* scores = reinterpret_cast<float*>(d + sl.d_scores);
    int32_t* nv = reinterpret_cast<int32_t*>(d + sl.d_nv);
    r = csa_index_scores(c, layer, n, req_ids, reinterpret_cast<const float*>(d + sl.qi),
                         reinterpret_cast<const float*>(d + sl.w), scores, sl.ld, nv, CSA_VARIANT_AUTO, stream);
    if (r == CSA_OK) r = csa_topk(scores, sl.ld, nv, n, k, idx, CSA_VARIANT_AUTO, stream);
  }
  if (r != CSA_OK) return r;
  e = cudaStreamWaitEvent(st, c->ev_q, 0);
  if (e != cudaSuccess) return cuda_fail(e, "decode step join");
  r = csa_hca_decode_attn(c, layer, n, req_ids, d + sl.q, idx, csa ? k : 0, sink, scale,
                          out_dev != nullptr ? out_dev : d + sl.d_out, d + sl.d_ws, sl.ws_bytes,
                          (csa_variant)(CSA_VARIANT_AUTO | (csa ? CSA_ATTN_STATE_READY : 0)), stream);
  if (r != CSA_OK) return r;
  if (out_dev == nullptr) {
    e = cudaMemcpyAsync(host_out, d + sl.d_out, (size_t)sl.out_bytes, cudaMemcpyDeviceToHost, st);
    if (e != cudaSuccess) return cuda_fail(e, "decode step output copy");
  }
  return CSA_OK;
}

// ---- a chunk of queries with causal visibility (prefill)

namespace {

struct ChunkLayout {
  int64_t snap, req, scores, nv, idx, ws, total, ld;
  size_t ws_bytes;
};

ChunkLayout chunk_layout(const csa_cache* c, int32_t layer, int32_t n, int32_t n_tok, int32_t k, csa_variant variant) {
  const Layout& L = c->L;
  const bool csa = layer < L.n_csa;
  const int64_t Q = (int64_t)n * n_tok;
  auto al = [](int64_t x) { return (x + 255) / 256 * 256; };
  ChunkLayout s{};
  int64_t o = 0;
  s.snap = o;   o += al((int64_t)n * L.ring_bytes);
  s.req = o;    o += al(Q * 4);
  s.ld = csa ? std::max<int64_t>((int64_t)L.max_pages_per_req * csa::kCsaPerPage, 128) : 0;
  s.scores = o; o += al(Q * s.ld * 4);
  s.nv = o;     o += al(csa ? Q * 4 : 0);
  s.idx = o;    o += al(csa ? Q * k * 4 : 0);
  s.ws_bytes = attn_split(L, (int32_t)Q, variant, true) ? csa::attn_workspace_bytes(L, layer, (int)Q, csa ? k : 0) : 0;
  s.ws = o;     o += al((int64_t)s.ws_bytes);
  s.total = o;
  return s;
}

bool chunk_shape_ok(const csa_cache* c, int32_t layer, int32_t n, int32_t n_tok, int32_t k, csa_variant variant,
                    std::string* why) {
  if (!layer_ok(c, layer)) { *why = "bad layer"; return false; }
  if (n < 1 || n > 65535) { *why = "n must be in [1, 65535]"; return false; }
  if (n_tok < 1 || n_tok > csa::kWindow) { *why = "n_tok must be in [1, 128]"; return false; }
  if ((int64_t)n * n_tok > 65535) { *why = "n * n_tok must be <= 65535"; return false; }
  if (layer < c->L.n_csa && (k < 1 || k > 8192)) { *why = "a CSA layer needs 1 <= k <= 8192"; return false; }
  if (variant < CSA_VARIANT_AUTO || variant > CSA_VARIANT_LOW_OCC) { *why = "bad variant"; return false; }
  return true;
}

}  // namespace

size_t csa_prefill_workspace_bytes(const csa_cache_t* c, int32_t layer, int32_t n, int32_t n_tok, int32_t k,
                                   csa_variant variant) {
  std::string why;
  if (!chunk_shape_ok(c, layer, n, n_tok, k, variant, &why)) return 0;
  return (size_t)chunk_layout(c, layer, n, n_tok, layer < c->L.n_csa ? k : 0, variant).total;
}

csa_status csa_prefill_chunk(csa_cache_t* c, int32_t layer, int32_t n, const int32_t* req_ids, int32_t n_tok,
                             const float* kv_cand, const float* kv_gate, const float* idx_cand,
                             const float* idx_gate, const void* q, const float* q_idx, const float* w, int32_t k,
                             const float* sink, float scale, void* out, int32_t* topk_out, void* workspace,
                             size_t workspace_bytes, csa_variant variant, csa_stream_t stream) {
  std::string why;
  if (!chunk_shape_ok(c, layer, n, n_tok, k, variant, &why)) return fail(CSA_ERR_ARG, why);
  const bool csa = layer < c->L.n_csa;
  if (!req_ids || !kv_cand || !kv_gate || !q || !sink || !out || !workspace) return fail(CSA_ERR_ARG, "NULL argument");
  if (csa && (!idx_cand || !idx_gate || !q_idx || !w)) return fail(CSA_ERR_ARG, "a CSA layer needs the index inputs");
  if (reinterpret_cast<uintptr_t>(workspace) % 256) return fail(CSA_ERR_ARG, "workspace must be 256-byte aligned");
  const int kk = csa ? k : 0;
  const ChunkLayout cl = chunk_layout(c, layer, n, n_tok, kk, variant);
  if (workspace_bytes < (size_t)cl.total) return fail(CSA_ERR_ARG, "workspace smaller than csa_prefill_workspace_bytes");
  const int32_t Q = n * n_tok;
  char* ws = static_cast<char*>(workspace);
  char* snap = ws + cl.snap;
  int32_t* req_exp = reinterpret_cast<int32_t*>(ws + cl.req);
  // the rings as they are before the chunk, and one request id per query
  cudaError_t e = csa::launch_chunk_prep(c->L, layer, n, req_ids, n_tok, req_exp, snap, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "chunk set-up launch");
  csa_status r = csa_compress_append(c, layer, n, req_ids, n_tok, kv_cand, kv_gate, idx_cand, idx_gate, stream);
  if (r != CSA_OK) return r;
  const ChunkQ cq{n_tok, snap};
  int32_t* idx = nullptr;
  if (csa) {
    idx = topk_out ? topk_out : reinterpret_cast<int32_t*>(ws + cl.idx);
    float* scores = reinterpret_cast<float*>(ws + cl.scores);
    int32_t* nv = reinterpret_cast<int32_t*>(ws + cl.nv);
    r = index_scores_impl(c, layer, Q, req_exp, q_idx, w, scores, cl.ld, nv, variant, stream, cq);
    if (r == CSA_OK) r = csa_topk(scores, cl.ld, nv, Q, k, idx, variant, stream);
    if (r != CSA_OK) return r;
  }
  return decode_attn_impl(c, layer, Q, req_exp, q, idx, kk, sink, scale, out, cl.ws_bytes ? ws + cl.ws : nullptr,
                          cl.ws_bytes, variant, stream, cq);
}

// ---- batch-invariant projection GEMM

static bool gemm_shape_ok(int32_t n_out, int32_t k_in, int32_t groups, std::string* why) {
  if (n_out < 1 || k_in < 1 || groups < 1) { *why = "n_out, k_in and groups must be >= 1"; return false; }
  if (groups > 65535) { *why = "groups must be <= 65535"; return false; }
  if (n_out % groups || k_in % groups) { *why = "groups must divide n_out and k_in"; return false; }
  if (groups > 1 && (n_out / groups) % 128) { *why = "a grouped weight needs a multiple of 128 rows per group"; return false; }
  if ((k_in / groups) % 8) { *why = "k_in / groups must be a multiple of 8"; return false; }
  return true;
}

size_t csa_gemm_weight_bytes(int32_t n_out, int32_t k_in, int32_t groups) {
  std::string why;
  if (!gemm_shape_ok(n_out, k_in, groups, &why)) return 0;
  return csa::gemm_weight_bytes(n_out, k_in, groups);
}

csa_status csa_gemm_pack_weight(const uint16_t* w_host, int32_t n_out, int32_t k_in, int32_t groups, void* w_dev,
                                size_t bytes) {
  std::string why;
  if (!gemm_shape_ok(n_out, k_in, groups, &why)) return fail(CSA_ERR_ARG, why);
  if (!w_host || !w_dev || reinterpret_cast<uintptr_t>(w_dev) % 16) return fail(CSA_ERR_ARG, "NULL or unaligned pointer");
  const size_t need = csa::gemm_weight_bytes(n_out, k_in, groups);
  if (bytes < need) return fail(CSA_ERR_CAPACITY, "w_dev smaller than csa_gemm_weight_bytes");
  std::vector<uint8_t> tiles;
  try {
    tiles.resize(need);
  } catch (...) {
    return fail(CSA_ERR_CAPACITY, "host allocation failed");
  }
  csa::gemm_pack_weight_host(w_host, n_out, k_in, groups, tiles.data());
  cudaError_t e = cudaMemcpy(w_dev, tiles.data(), need, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(packed weight)");
  return CSA_OK;
}

size_t csa_gemm_workspace_bytes(int32_t n_out, int32_t k_in, int32_t groups, int32_t n_tok) {
  std::string why;
  if (!gemm_shape_ok(n_out, k_in, groups, &why) || n_tok < 1 || n_tok > csa::gemm_max_tokens()) return 0;
  const int sms = sm_count();
  if (sms <= 0) return 0;
  return csa::gemm_workspace_bytes(n_out, k_in, groups, n_tok, sms);
}

csa_status csa_gemm_bf16(const void* w_packed, int32_t n_out, int32_t k_in, int32_t groups, const uint16_t* x,
                         int32_t n_tok, int32_t n_seg, const csa_gemm_out* segs, void* workspace,
                         size_t workspace_bytes, csa_stream_t stream) {
  std::string why;
  if (!gemm_shape_ok(n_out, k_in, groups, &why)) return fail(CSA_ERR_ARG, why);
  if (n_tok < 0 || n_tok > csa::gemm_max_tokens()) return fail(CSA_ERR_ARG, "n_tok must be in [0, 256]");
  if (n_seg < 1 || n_seg > csa::kGemmMaxSeg || !segs) return fail(CSA_ERR_ARG, "n_seg must be in [1, 8]");
  csa::GemmOut out{};
  out.n_seg = n_seg;
  int rows = 0;
  for (int s = 0; s < n_seg; ++s) {
    if (segs[s].rows < 1 || !segs[s].y) return fail(CSA_ERR_ARG, "every output segment needs rows >= 1 and y");
    rows += segs[s].rows;
    out.seg_end[s] = rows;
    out.y[s] = segs[s].y;
    if (segs[s].bf16) out.bf16_mask |= 1u << s;
  }
  if (rows != n_out) return fail(CSA_ERR_ARG, "the segments' rows must add up to n_out");
  if (n_tok == 0) return CSA_OK;
  if (!w_packed || !x || !workspace) return fail(CSA_ERR_ARG, "NULL argument");
  if (reinterpret_cast<uintptr_t>(w_packed) % 16 || reinterpret_cast<uintptr_t>(workspace) % 256)
    return fail(CSA_ERR_ARG, "w_packed must be 16-byte and workspace 256-byte aligned");
  const int sms = sm_count();
  if (sms <= 0) return fail(CSA_ERR_CUDA, "cannot query the SM count");
  if (workspace_bytes < csa::gemm_workspace_bytes(n_out, k_in, groups, n_tok, sms))
    return fail(CSA_ERR_ARG, "workspace smaller than csa_gemm_workspace_bytes");
  cudaError_t e = csa::launch_gemm_bf16(w_packed, n_out, k_in, groups, x, n_tok, out, workspace, sms,
                                        (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "gemm launch");
  return CSA_OK;
}

csa_status csa_gemm_check_device_error(csa_stream_t stream) {
  int32_t code = 0, detail = 0;
  cudaError_t e = csa::gemm_read_error(&code, &detail, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "gemm error word");
  if (code == 0) return CSA_OK;
  char msg[120];
  snprintf(msg, sizeof msg, "device: a GEMM pipeline wait gave up (row tile %d)", detail);
  return fail(CSA_ERR_DEVICE_TIMEOUT, msg);
}

csa_status csa_debug_wait_timeout(csa_cache_t* c, int32_t limit_us, csa_stream_t stream) {
  if (!c) return fail(CSA_ERR_ARG, "cache is NULL");
  if (limit_us < 1 || limit_us > 1000000) return fail(CSA_ERR_ARG, "limit_us must be in [1, 1000000]");
  cudaError_t e = csa::launch_wait_probe(c->L, (uint64_t)limit_us * 1000ull, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "wait probe launch");
  return CSA_OK;
}

size_t csa_debug_row_bytes(const csa_cache_t* c, int32_t region) {
  if (!c) return 0;
  const Layout& L = c->L;
  const bool f32 = L.fmt == csa::kFmtF32;
  if (region == CSA_REGION_KV || region == CSA_REGION_WINDOW) return f32 ? (size_t)L.D * 4 : (size_t)(L.D + L.R + 4);
  if (region == CSA_REGION_INDEX) return f32 ? (size_t)L.dI * 4 : (size_t)(L.dI / 2 + L.dI / 32);
  return 0;
}

int64_t csa_debug_get_length(csa_cache_t* c, int32_t layer, int32_t req) {
  if (!layer_ok(c, layer) || req < 0 || req >= c->L.max_req) return -1;
  int64_t v = -1;
  if (cudaMemcpy(&v, c->L.lengths() + (int64_t)layer * c->L.max_req + req, 8, cudaMemcpyDeviceToHost) != cudaSuccess)
    return -1;
  return v;
}

csa_status csa_debug_set_length(csa_cache_t* c, int32_t layer, int32_t req, int64_t len) {
  if (!layer_ok(c, layer) || req < 0 || req >= c->L.max_req) return fail(CSA_ERR_ARG, "bad layer/request");
  if (len < 0 || len > (int64_t)c->req_pages[req].size() * csa::kPageTokens)
    return fail(CSA_ERR_CAPACITY, "length beyond the request's capacity");
  cudaError_t e = cudaMemcpy(c->L.lengths() + (int64_t)layer * c->L.max_req + req, &len, 8, cudaMemcpyHostToDevice);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemcpy(length)");
  return CSA_OK;
}

// Copy `bytes` between host and device in the requested direction.
static cudaError_t xfer(void* dev, void* host, size_t bytes, bool write) {
  return write ? cudaMemcpy(dev, host, bytes, cudaMemcpyHostToDevice)
               : cudaMemcpy(host, dev, bytes, cudaMemcpyDeviceToHost);
}

// Rows are moved page by page: a whole page section is copied to host
// memory, rows are packed or unpacked there, and (for writes) the section is
// copied back.
csa_status csa_debug_rows(csa_cache_t* c, int32_t layer, int32_t req, int32_t region, int64_t first,
                          int64_t count, void* host, int32_t write) {
  if (!layer_ok(c, layer) || req < 0 || req >= c->L.max_req) return fail(CSA_ERR_ARG, "bad layer/request");
  if (!host || first < 0 || count < 0) return fail(CSA_ERR_ARG, "bad rows");
  const Layout& L = c->L;
  const bool is_csa = layer < L.n_csa;
  const int64_t fp8b = L.kv_fp8_bytes, bfb = L.kv_bf16_bytes;
  const size_t rb = csa_debug_row_bytes(c, region);
  if (rb == 0) return fail(CSA_ERR_ARG, "bad region");
  if (region == CSA_REGION_INDEX && !is_csa) return fail(CSA_ERR_ARG, "index keys exist on CSA layers only");
  auto& held = c->req_pages[req];
  char* h = static_cast<char*>(host);
  const bool wr = write != 0;
  const bool f32 = L.fmt == csa::kFmtF32;
  if (region == CSA_REGION_WINDOW) {
    char* st = L.state(req, layer);
    std::vector<char> ring(L.ring_bytes);
    cudaError_t e = xfer(st, ring.data(), L.ring_bytes, false);
    if (e != cudaSuccess) return cuda_fail(e, "debug ring read");
    for (int64_t r = 0; r < count; ++r) {
      const int slot = (int)((first + r) % csa::kWindow);
      char* row = h + r * rb;
      if (f32) {
        char* a = ring.data() + (int64_t)slot * rb;
        if (wr) memcpy(a, row, rb); else memcpy(row, a, rb);
        continue;
      }
      char* a = ring.data() + L.ring_fp8 + slot * fp8b;
      char* b = ring.data() + L.ring_bf16 + slot * bfb;
      char* s = ring.data() + L.ring_scale + slot * 4;
      if (wr) { memcpy(a, row, fp8b); memcpy(b, row + fp8b, bfb); memcpy(s, row + fp8b + bfb, 4); }
      else { memcpy(row, a, fp8b); memcpy(row + fp8b, b, bfb); memcpy(row + fp8b + bfb, s, 4); }
    }
    if (wr) {
      e = xfer(st, ring.data(), L.ring_bytes, true);
      if (e != cudaSuccess) return cuda_fail(e, "debug ring write");
    }
    return CSA_OK;
  }
  const int64_t per_pg = L.rows_per_page(layer);
  const int64_t sec = is_csa ? L.pg_csa_bytes : L.pg_hca_bytes;
  std::vector<char> buf(sec);
  const int CH = L.dI / 32;
  int64_t r = 0;
  while (r < count) {
    const int64_t j0 = first + r;
    const int64_t lp = j0 / per_pg;
    if (lp >= (int64_t)held.size()) return fail(CSA_ERR_ARG, "entry beyond the request's pages");
    char* pp = L.page(held[lp], layer);
    cudaError_t e = xfer(pp, buf.data(), sec, false);
    if (e != cudaSuccess) return cuda_fail(e, "debug page read");
    for (; r < count && (first + r) / per_pg == lp; ++r) {
      const int s = (int)((first + r) % per_pg);
      char* row = h + r * rb;
      if (f32) {   // fp32 rows [P][D] then (CSA) fp32 keys [P][d_I]
        char* a = buf.data() + (region == CSA_REGION_KV ? 0 : L.pg_idx_f32) + (int64_t)s * rb;
        if (wr) memcpy(a, row, rb); else memcpy(row, a, rb);
        continue;
      }
      if (region == CSA_REGION_KV) {
        char* a = buf.data() + s * fp8b;
        char* b = buf.data() + (is_csa ? L.pg_csa_bf16 : L.pg_hca_bf16) + s * bfb;
        char* sc = buf.data() + (is_csa ? L.pg_csa_scale : L.pg_hca_scale) + s * 4;
        if (wr) { memcpy(a, row, fp8b); memcpy(b, row + fp8b, bfb); memcpy(sc, row + fp8b + bfb, 4); }
        else { memcpy(row, a, fp8b); memcpy(row + fp8b, b, bfb); memcpy(row + fp8b + bfb, sc, 4); }
      } else {
        char* tile = buf.data() + L.pg_idx_codes;
        for (int ch = 0; ch < L.CHs; ++ch) {
          char* cp = tile + L.idx_code_off(s, ch);
          if (ch < CH) { if (wr) memcpy(cp, row + ch * 16, 16); else memcpy(row + ch * 16, cp, 16); }
          else if (wr) memset(cp, 0, 16);
        }
        char* sf = buf.data() + L.pg_idx_sf;
        for (int k = 0; k < 4; ++k) {
          char* sp = sf + Layout::idx_sf_off(s, k);
          if (k < CH) { if (wr) *sp = row[L.dI / 2 + k]; else row[L.dI / 2 + k] = *sp; }
          else if (wr) *sp = 127;
        }
      }
    }
    if (wr) {
      e = xfer(pp, buf.data(), sec, true);
      if (e != cudaSuccess) return cuda_fail(e, "debug page write");
    }
  }
  return CSA_OK;
}

}  // extern "C"
