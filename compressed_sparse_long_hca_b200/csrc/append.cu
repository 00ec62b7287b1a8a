// Token-level compressor and cache write (csa_compress_append).
//
// Page "V4终于终于终于终于是来了", section "CSA——压缩稀疏注意力": a token-level
// compressor turns every 4 tokens' KV into one entry, and the lightning
// indexer keeps compressed index keys; section "HCA——重度压缩注意力": HCA
// compresses 128 tokens into one entry, the state cache keeps the latest 128
// raw tokens and the unfinished tails, the classic cache keeps entries in
// 128-token blocks.  Page "深度解读DeepSeek V4 看清Benchmark以外的三个范式创新",
// section 01 "混合注意力的精细解剖": CSA windows overlap so that meaning is not cut
// at block edges.
//
// Entry j of CSA pools tokens [4j-4, 4j+4) (those >= 0), of HCA tokens
// [128j, 128j+128); per channel the weights are softmax over the window's
// tokens of (gate logit + position bias of the token's window slot).
//
// General call (any n_tok): three launches, stream-ordered:
//   1. entries: every entry completed by the new tokens (reads tails + input)
//   2. tokens:  window-ring rows and tail slots of the new tokens
//   3. length:  L += n_tok
// Launch 1 reads the tails before launch 2 overwrites them.
// Decode call (n_tok == 1): one launch, two CTAs per request (the token's
// ring row and tail slot; the entry it completes, if any).  With one new
// token the tail slot it overwrites is never one the completed entry reads
// (the entry's older tokens sit in the other slots of the ring), so the two
// roles can run concurrently.  Both CTAs of a request read its length first
// and then take a ticket of the request; the second one advances the length
// (with the value both read) and resets the ticket for the next call.  The
// token CTA loads its inputs before the request's state, so that the two
// round trips overlap.
#include "common.cuh"

namespace csa {

struct AppendArgs {
  Layout L;
  int layer;
  int n;
  const int32_t* req_ids;
  int n_tok;
  const float* c;
  const float* z;
  const float* ci;
  const float* zi;
};

// Fetch channel `ch` of token `tau` (which the entry's window needs) from the
// new-token input (tau >= L0) or from the request's tail ring.
__device__ __forceinline__ void fetch_tok(const AppendArgs& a, int i, int64_t L0, int64_t tau, int ch,
                                          int dim, const float* in_c, const float* in_z,
                                          const float* tail_c, const float* tail_z, int ring,
                                          float& c, float& z) {
  if (tau >= L0) {
    const int64_t o = ((int64_t)i * a.n_tok + (tau - L0)) * dim + ch;
    c = in_c[o];
    z = in_z[o];
  } else {
    const int64_t o = (int64_t)(tau % ring) * dim + ch;
    c = tail_c[o];
    z = tail_z[o];
  }
}

__device__ __forceinline__ bool load_request(const AppendArgs& a, int i, int& req, int64_t& L0) {
  req = a.req_ids[i];
  if (req < 0 || req >= a.L.max_req) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_err(a.L, kErrBounds, i);
    return false;
  }
  L0 = a.L.lengths()[(int64_t)a.layer * a.L.max_req + req];
  const int64_t cap = (int64_t)a.L.capacity()[req] * kPageTokens;
  if (L0 + a.n_tok > cap) {
    if (threadIdx.x == 0 && blockIdx.y == 0) set_err(a.L, kErrCapacity, req);
    return false;
  }
  return true;
}

// ---------------------------------------------------------------- launch 1

__device__ void csa_entries_body(const AppendArgs& a, int i, int req, int64_t L0, int y0, int ystride, float* sm) {
  const Layout& L = a.L;
  const int D = L.D, R = L.R, dI = L.dI;
  float* row = sm;            // [D]
  float* key = sm + D;        // [dI]
  float* red = key + dI;      // [32]
  const int64_t n_done = (L0 + a.n_tok) / kCsaM;    // entries complete after the call
  const float* tc = reinterpret_cast<const float*>(L.tail(req, a.layer));
  const float* tz = tc + kCsaWin * D;
  const float* tci = tz + kCsaWin * D;
  const float* tzi = tci + kCsaWin * dI;
  const float* bkv = L.bpos_csa(a.layer);
  const float* bix = L.bpos_idx(a.layer);
  for (int64_t j = L0 / kCsaM + y0; j < n_done; j += ystride) {
    const int64_t t0 = kCsaM * j - kCsaM;          // first window token (may be < 0)
    for (int ch = threadIdx.x; ch < D + dI; ch += blockDim.x) {
      const bool is_kv = ch < D;
      const int cc = is_kv ? ch : ch - D;
      const int dim = is_kv ? D : dI;
      const float* b = is_kv ? bkv : bix;
      float cv[kCsaWin], lg[kCsaWin];
      float mx = -INFINITY;
      for (int s = 0; s < kCsaWin; ++s) {
        const int64_t tau = t0 + s;
        if (tau < 0) { lg[s] = -INFINITY; cv[s] = 0.f; continue; }
        float c, z;
        fetch_tok(a, i, L0, tau, cc, dim, is_kv ? a.c : a.ci, is_kv ? a.z : a.zi,
                  is_kv ? tc : tci, is_kv ? tz : tzi, kCsaWin, c, z);
        cv[s] = c;
        lg[s] = z + b[s * dim + cc];
        mx = fmaxf(mx, lg[s]);
      }
      float num = 0.f, den = 0.f;
      for (int s = 0; s < kCsaWin; ++s) {
        if (lg[s] == -INFINITY) continue;
        const float e = expf(lg[s] - mx);
        den += e;
        num = fmaf(e, cv[s], num);
      }
      const float v = __fdiv_rn(num, den);
      if (is_kv) row[cc] = v; else key[cc] = v;
    }
    __syncthreads();
    for (int p = threadIdx.x; p < R / 2; p += blockDim.x)
      rope_pair(row[D - R + 2 * p], row[D - R + 2 * p + 1], L.theta()[p], kCsaM * j);
    __syncthreads();
    if (L.fmt == kFmtF32) {
      store_f32_row(row, D, L.entry_row_f32(req, a.layer, j));
      store_f32_row(key, dI, L.index_key_f32(req, a.layer, j));
    } else {
      const int s = (int)(j % kCsaPerPage);
      char* pp = L.page(L.page_table(req)[j / kCsaPerPage], a.layer);
      store_kv_row(row, D, R, reinterpret_cast<uint8_t*>(pp) + (int64_t)s * (D - R),
                   reinterpret_cast<uint16_t*>(pp + L.pg_csa_bf16) + (int64_t)s * R,
                   reinterpret_cast<float*>(pp + L.pg_csa_scale) + s, red);
      store_index_key(L, key, s, reinterpret_cast<uint8_t*>(pp + L.pg_idx_codes),
                      reinterpret_cast<uint8_t*>(pp + L.pg_idx_sf));
    }
    __syncthreads();
  }
}

__device__ void hca_entries_body(const AppendArgs& a, int i, int req, int64_t L0, int y0, int ystride, float* sm) {
  const Layout& L = a.L;
  const int D = L.D, R = L.R;
  float* row = sm;
  float* red = sm + D;
  const int64_t n_done = (L0 + a.n_tok) / kHcaM;
  const float* tc = reinterpret_cast<const float*>(L.tail(req, a.layer));
  const float* tz = tc + kHcaM * D;
  const float* b = L.bpos_hca(a.layer - L.n_csa);
  for (int64_t j = L0 / kHcaM + y0; j < n_done; j += ystride) {
    const int64_t t0 = kHcaM * j;
    for (int ch = threadIdx.x; ch < D; ch += blockDim.x) {
      float mx = -INFINITY;
      for (int s = 0; s < kHcaM; ++s) {
        float c, z;
        fetch_tok(a, i, L0, t0 + s, ch, D, a.c, a.z, tc, tz, kHcaM, c, z);
        mx = fmaxf(mx, z + b[s * D + ch]);
      }
      float num = 0.f, den = 0.f;
      for (int s = 0; s < kHcaM; ++s) {
        float c, z;
        fetch_tok(a, i, L0, t0 + s, ch, D, a.c, a.z, tc, tz, kHcaM, c, z);
        const float e = expf(z + b[s * D + ch] - mx);
        den += e;
        num = fmaf(e, c, num);
      }
      row[ch] = __fdiv_rn(num, den);
    }
    __syncthreads();
    for (int p = threadIdx.x; p < R / 2; p += blockDim.x)
      rope_pair(row[D - R + 2 * p], row[D - R + 2 * p + 1], L.theta()[p], kHcaM * j);
    __syncthreads();
    if (L.fmt == kFmtF32) {
      store_f32_row(row, D, L.entry_row_f32(req, a.layer, j));
    } else {
      const int s = (int)(j % kHcaPerPage);
      char* pp = L.page(L.page_table(req)[j / kHcaPerPage], a.layer);
      store_kv_row(row, D, R, reinterpret_cast<uint8_t*>(pp) + (int64_t)s * (D - R),
                   reinterpret_cast<uint16_t*>(pp + L.pg_hca_bf16) + (int64_t)s * R,
                   reinterpret_cast<float*>(pp + L.pg_hca_scale) + s, red);
    }
    __syncthreads();
  }
}

__global__ void __launch_bounds__(256) csa_entries_kernel(AppendArgs a) {
  extern __shared__ float sm[];
  int req;
  int64_t L0;
  if (!load_request(a, blockIdx.x, req, L0)) return;
  csa_entries_body(a, blockIdx.x, req, L0, blockIdx.y, gridDim.y, sm);
}

__global__ void __launch_bounds__(256) hca_entries_kernel(AppendArgs a) {
  extern __shared__ float sm[];
  int req;
  int64_t L0;
  if (!load_request(a, blockIdx.x, req, L0)) return;
  hca_entries_body(a, blockIdx.x, req, L0, blockIdx.y, gridDim.y, sm);
}

// ---------------------------------------------------------------- launch 2

__device__ void tokens_body(const AppendArgs& a, int i, int y0, int ystride, float* sm) {
  const Layout& L = a.L;
  const int D = L.D, R = L.R, dI = L.dI;
  const bool csa = a.layer < L.n_csa;
  float* row = sm;
  float* red = sm + D;
  int req;
  int64_t L0;
  if (!load_request(a, i, req, L0)) return;
  const int64_t L1 = L0 + a.n_tok;
  char* st = L.state(req, a.layer);
  // window ring rows for positions max(L0, L1-128) .. L1-1
  const int64_t r0 = L1 - kWindow > L0 ? L1 - kWindow : L0;
  for (int64_t pos = r0 + y0; pos < L1; pos += ystride) {
    const float* src = a.c + ((int64_t)i * a.n_tok + (pos - L0)) * D;
    for (int d = threadIdx.x; d < D; d += blockDim.x) row[d] = src[d];
    __syncthreads();
    for (int p = threadIdx.x; p < R / 2; p += blockDim.x)
      rope_pair(row[D - R + 2 * p], row[D - R + 2 * p + 1], L.theta()[p], pos);
    __syncthreads();
    const int slot = (int)(pos % kWindow);
    if (L.fmt == kFmtF32)
      store_f32_row(row, D, L.ring_row_f32(req, a.layer, slot));
    else
      store_kv_row(row, D, R, reinterpret_cast<uint8_t*>(st + L.ring_fp8) + (int64_t)slot * (D - R),
                   reinterpret_cast<uint16_t*>(st + L.ring_bf16) + (int64_t)slot * R,
                   reinterpret_cast<float*>(st + L.ring_scale) + slot, red);
    __syncthreads();
  }
  // tail slots
  float* tail = reinterpret_cast<float*>(L.tail(req, a.layer));
  const int ring = csa ? kCsaWin : kHcaM;
  int64_t t_lo = csa ? L1 - kCsaWin : (L1 / kHcaM) * kHcaM;
  if (t_lo < L0) t_lo = L0;
  for (int64_t pos = t_lo + y0; pos < L1; pos += ystride) {
    const int slot = (int)(pos % ring);
    const int64_t src = (int64_t)i * a.n_tok + (pos - L0);
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
      tail[(int64_t)slot * D + d] = a.c[src * D + d];
      tail[(int64_t)ring * D + (int64_t)slot * D + d] = a.z[src * D + d];
    }
    if (csa) {
      float* ti = tail + 2 * (int64_t)ring * D;
      for (int d = threadIdx.x; d < dI; d += blockDim.x) {
        ti[(int64_t)slot * dI + d] = a.ci[src * dI + d];
        ti[(int64_t)ring * dI + (int64_t)slot * dI + d] = a.zi[src * dI + d];
      }
    }
  }
}

__global__ void __launch_bounds__(256) tokens_kernel(AppendArgs a) {
  extern __shared__ float sm[];
  tokens_body(a, blockIdx.x, blockIdx.y, gridDim.y, sm);
}

// ---------------------------------------------------------------- launch 3

__global__ void length_kernel(AppendArgs a) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= a.n) return;
  const int req = a.req_ids[i];
  if (req < 0 || req >= a.L.max_req) return;
  int64_t* len = a.L.lengths() + (int64_t)a.layer * a.L.max_req + req;
  const int64_t cap = (int64_t)a.L.capacity()[req] * kPageTokens;
  if (*len + a.n_tok <= cap) *len += a.n_tok;
}

// ---------------------------------------------------------------- decode: one launch

// The decode token (n_tok == 1) of request slot i: its ring row and tail
// slot.  One thread per channel (blockDim >= D).  The token's inputs and
// RoPE frequencies are loaded before the request's state; returns false
// when the request is skipped.
__device__ bool token1_body(const AppendArgs& a, int i, float* sm, int& req, int64_t& L0) {
  const Layout& L = a.L;
  const int D = L.D, R = L.R, dI = L.dI;
  const bool csa = a.layer < L.n_csa;
  float* row = sm;
  float* red = sm + D;
  const int t = threadIdx.x;
  const float* c = a.c + (int64_t)i * D;
  const float* z = a.z + (int64_t)i * D;
  const float c0 = t < D ? c[t] : 0.f;
  const float z0 = t < D ? z[t] : 0.f;
  float ci0 = 0.f, zi0 = 0.f;
  if (csa && t < dI) {
    ci0 = a.ci[(int64_t)i * dI + t];
    zi0 = a.zi[(int64_t)i * dI + t];
  }
  const double th = t < R / 2 ? L.theta()[t] : 0.0;
  if (!load_request(a, i, req, L0)) return false;
  const int64_t pos = L0;
  if (t < D) row[t] = c0;
  __syncthreads();
  if (t < R / 2) rope_pair(row[D - R + 2 * t], row[D - R + 2 * t + 1], th, pos);
  __syncthreads();
  char* st = L.state(req, a.layer);
  const int slot = (int)(pos % kWindow);
  if (L.fmt == kFmtF32)
    store_f32_row(row, D, L.ring_row_f32(req, a.layer, slot));
  else
    store_kv_row(row, D, R, reinterpret_cast<uint8_t*>(st + L.ring_fp8) + (int64_t)slot * (D - R),
                 reinterpret_cast<uint16_t*>(st + L.ring_bf16) + (int64_t)slot * R,
                 reinterpret_cast<float*>(st + L.ring_scale) + slot, red);
  // tail slot (an HCA block completed by this token needs no tail)
  if (csa || (pos + 1) % kHcaM != 0) {
    float* tail = reinterpret_cast<float*>(L.tail(req, a.layer));
    const int ring = csa ? kCsaWin : kHcaM;
    const int ts = (int)(pos % ring);
    if (t < D) { tail[(int64_t)ts * D + t] = c0; tail[(int64_t)ring * D + (int64_t)ts * D + t] = z0; }
    if (csa && t < dI) {
      float* ti = tail + 2 * (int64_t)ring * D;
      ti[(int64_t)ts * dI + t] = ci0;
      ti[(int64_t)ring * dI + (int64_t)ts * dI + t] = zi0;
    }
  }
  return true;
}

// grid (n, 2): blockIdx.y 0 = the token's ring row and tail slot, 1 = the
// entry it completes (if any).  n_tok == 1, request slots distinct.  One
// thread per channel of the entry (D + d_I on CSA layers, D on HCA), so that
// every channel's window loads are in flight at once.
__global__ void __launch_bounds__(640) append_decode_kernel(AppendArgs a) {
  extern __shared__ float sm[];
  const Layout& L = a.L;
  const int i = blockIdx.x;
  int req;
  int64_t L0;
  bool ok;
  if (blockIdx.y == 0) {
    ok = token1_body(a, i, sm, req, L0);
  } else {
    ok = load_request(a, i, req, L0);
    if (ok) {
      if (a.layer < L.n_csa) csa_entries_body(a, i, req, L0, 0, 1, sm);
      else hca_entries_body(a, i, req, L0, 0, 1, sm);
    }
  }
  if (!ok) return;   // both CTAs of the request skip it alike
  // both CTAs of the request have read its length; the second advances it
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    int32_t* tk = L.ticket(a.layer, req);
    if (atomicAdd(tk, 1) == 1) {
      *tk = 0;
      L.lengths()[(int64_t)a.layer * L.max_req + req] = L0 + a.n_tok;
    }
  }
}

cudaError_t launch_append(const Layout& L, int layer, int n, const int32_t* req_ids, int n_tok,
                          const float* c, const float* z, const float* ci, const float* zi,
                          cudaStream_t st) {
  AppendArgs a{L, layer, n, req_ids, n_tok, c, z, ci, zi};
  const bool csa = layer < L.n_csa;
  const int threads = 256;
  if (n_tok == 1) {
    const size_t sm = (size_t)(L.D + (csa ? L.dI : 0) + 32) * sizeof(float);
    const int dec_threads = (L.D + (csa ? L.dI : 0) + 31) / 32 * 32;   // <= 640
    append_decode_kernel<<<dim3(n, 2), dec_threads, sm, st>>>(a);
    note_launch();
    return cudaGetLastError();
  }
  // entries completed by n_tok new tokens: at most n_tok/m + 1 per request
  const int64_t emax = csa ? n_tok / kCsaM + 1 : n_tok / kHcaM + 1;
  dim3 g1(n, (unsigned)(emax < 1024 ? emax : 1024));
  if (csa) {
    const size_t sm = (size_t)(L.D + L.dI + 32) * sizeof(float);
    csa_entries_kernel<<<g1, threads, sm, st>>>(a);
    note_launch();
  } else {
    const size_t sm = (size_t)(L.D + 32) * sizeof(float);
    hca_entries_kernel<<<g1, threads, sm, st>>>(a);
    note_launch();
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int rows = n_tok < kWindow ? n_tok : kWindow;
  dim3 g2(n, (unsigned)rows);
  tokens_kernel<<<g2, threads, (size_t)(L.D + 32) * sizeof(float), st>>>(a);
  note_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  length_kernel<<<(n + 127) / 128, 128, 0, st>>>(a);
  note_launch();
  return cudaGetLastError();
}

// Set-up of a chunk of queries (csa_prefill_chunk), before the chunk's
// append: block b copies request req_ids[b]'s window ring (the rows the
// append is about to overwrite are still the pre-chunk ones) to
// snap + b * ring_bytes and writes the request id once per query of the
// chunk into req_exp[b * n_tok .. b * n_tok + n_tok - 1].
__global__ void __launch_bounds__(256) chunk_prep_kernel(Layout L, int layer, const int32_t* req_ids, int n_tok,
                                                       int32_t* req_exp, char* snap) {
  const int b = blockIdx.x;
  const int req = req_ids[b];
  for (int j = threadIdx.x; j < n_tok; j += blockDim.x) req_exp[(int64_t)b * n_tok + j] = req;
  if (req < 0 || req >= L.max_req) return;       // the append reports the bad id
  const uint4* src = reinterpret_cast<const uint4*>(L.state(req, layer));
  uint4* dst = reinterpret_cast<uint4*>(snap + (int64_t)b * L.ring_bytes);
  for (int64_t x = threadIdx.x; x < L.ring_bytes / 16; x += blockDim.x) dst[x] = src[x];
}

cudaError_t launch_chunk_prep(const Layout& L, int layer, int n, const int32_t* req_ids, int n_tok, int32_t* req_exp,
                              char* snap, cudaStream_t st) {
  chunk_prep_kernel<<<n, 256, 0, st>>>(L, layer, req_ids, n_tok, req_exp, snap);
  note_launch();
  return cudaGetLastError();
}

// 16-byte chunks from src to dst (csa_decode_step: the step's small inputs
// read straight from page-locked host memory over the bus, one chunk per
// thread, every load in flight at once).
__global__ void __launch_bounds__(256) copy16_kernel(const uint4* src, uint4* dst, int64_t n16) {
  for (int64_t x = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; x < n16; x += (int64_t)gridDim.x * blockDim.x)
    dst[x] = src[x];
}

cudaError_t launch_copy16(const void* src, void* dst, size_t bytes, cudaStream_t st) {
  const int64_t n16 = (int64_t)(bytes / 16);
  if (n16 == 0) return cudaSuccess;
  const int64_t blocks = (n16 + 255) / 256;
  copy16_kernel<<<(unsigned)(blocks < 4096 ? blocks : 4096), 256, 0, st>>>(static_cast<const uint4*>(src),
                                                                         static_cast<uint4*>(dst), n16);
  note_launch();
  return cudaGetLastError();
}

}  // namespace csa
