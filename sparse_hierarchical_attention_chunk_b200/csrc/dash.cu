// C ABI of the DashAttention forward path (declared in include/dash.h).
//
// Host side only: argument validation, tensor-map encoding for TMA, kernel
// selection and launch on the caller's stream.  One translation unit, so
// every kernel shares the device error word that bounded waits set.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>
#include <math.h>
#include <stdint.h>
#include <string.h>

#include "dash.h"
#include "dash_common.cuh"
#include "tmap.cuh"
#include "summarize.cuh"
#include "route.cuh"
#include "route_tc.cuh"
#include "route_topk.cuh"
#include "attn_bwd.cuh"
#include "attn_bwd_tc.cuh"
#include "route_bwd.cuh"
#include "attn_tc.cuh"
#include "attn_f32.cuh"
#include "decode.cuh"

namespace {

using bf16 = __nv_bfloat16;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_problem(const dash_problem* p, bool decode) {
  if (!p) return DASH_ERR_INVALID_ARG;
  if (p->batch < 1 || p->n_q_heads < 1 || p->n_kv_heads < 1 || p->seq_len < 1)
    return DASH_ERR_INVALID_ARG;
  if (p->n_q_heads % p->n_kv_heads != 0) return DASH_ERR_INVALID_ARG;
  if (p->head_dim != 64 && p->head_dim != 128) return DASH_ERR_INVALID_ARG;
  if (p->chunk != 64 && p->chunk != 128) return DASH_ERR_INVALID_ARG;
  if (!decode && p->seq_len % p->chunk != 0) return DASH_ERR_INVALID_ARG;
  if (!(p->alpha > 1.f) || !(p->alpha <= 2.f)) return DASH_ERR_INVALID_ARG;
  if (!(p->gamma > 0.f) || !isfinite(p->gamma)) return DASH_ERR_INVALID_ARG;
  if (!(p->sigma >= 0.f) || !isfinite(p->sigma)) return DASH_ERR_INVALID_ARG;
  if (p->dtype != DASH_F32 && p->dtype != DASH_BF16) return DASH_ERR_INVALID_ARG;
  if (p->estimate_diagonal != 0 && p->estimate_diagonal != 1) return DASH_ERR_INVALID_ARG;
  // sizes must fit the 32-bit row indices used by the kernels and TMA
  const long long rows = (long long)p->batch * p->n_q_heads * p->seq_len;
  if (rows > (1ll << 31) - 1) return DASH_ERR_UNSUPPORTED;
  return DASH_OK;
}

int n_chunks(const dash_problem* p) { return (p->seq_len + p->chunk - 1) / p->chunk; }

// A failed runtime call (bad launch configuration, attribute, ...) leaves
// its code in the runtime's last-error slot; take it out so it is not
// reported again by an unrelated later call.  (A sticky device fault cannot
// be cleared this way and keeps failing every call, as it should.)
int cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return DASH_OK;
  (void)cudaGetLastError();
  return DASH_ERR_CUDA;
}

using dash::make_tmap;

template <int CHUNK, int D>
int run_attn_tc(const dash_problem* p, const void* Q, const void* K, const void* V,
                const float* w, const uint32_t* mask, void* O, float* lse, bool packed,
                cudaStream_t st) {
  const int G = p->n_q_heads / p->n_kv_heads;
  const int P = 128 / G;
  const uint64_t d = (uint64_t)D;
  CUtensorMap tq, tk, tv;
  {
    // Q viewed as (d, head, position): a box {64, G, P} lands position-major,
    // shared-memory row r = p * G + h
    const uint64_t dims[3] = {d, (uint64_t)p->batch * p->n_q_heads, (uint64_t)p->seq_len};
    const uint64_t str[2] = {(uint64_t)p->seq_len * d * 2, d * 2};
    const uint32_t box[3] = {64, (uint32_t)G, (uint32_t)P};
    if (!make_tmap(&tq, Q, 3, dims, str, box)) return DASH_ERR_CUDA;
  }
  {
    const uint64_t dims[2] = {d, (uint64_t)p->batch * p->n_kv_heads * p->seq_len};
    const uint64_t str[1] = {d * 2};
    const uint32_t box[2] = {64, (uint32_t)CHUNK};   // one key block per chunk
    if (!make_tmap(&tk, K, 2, dims, str, box)) return DASH_ERR_CUDA;
    if (!make_tmap(&tv, V, 2, dims, str, box)) return DASH_ERR_CUDA;
  }
  dash::AttnParams prm;
  prm.w = w;
  prm.mask = mask;
  prm.packed = packed ? 1 : 0;
  prm.O = static_cast<bf16*>(O);
  prm.lse = lse;
  prm.n_q = p->n_q_heads;
  prm.n_kv = p->n_kv_heads;
  prm.seq = p->seq_len;
  prm.chunk = p->chunk;
  prm.n_c = n_chunks(p);
  prm.nw = (prm.n_c + 31) / 32;
  prm.G = G;
  prm.P = P;
  prm.n_ctiles = p->seq_len / (2 * P);       // two 128-row tiles per CTA
  prm.n_bg = p->batch * p->n_kv_heads;
  prm.sigma = p->sigma;
  prm.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  return cuda_status(dash::launch_attn_tc<CHUNK, D>(tq, tk, tv, prm, st));
}

// Stage 2 backward on tcgen05: bf16, d = 128, G in {4, 8, 16}.
bool attn_bwd_tc_applies(const dash_problem* p) {
  const int G = p->n_q_heads / p->n_kv_heads;
  return p->dtype == DASH_BF16 && p->head_dim == 128 && (G == 4 || G == 8 || G == 16);
}

// The split count a test forced with dash_selftest_bwd_split (0: automatic).
int g_bwd_split_forced = 0;

// The backward's workspace layout, with a forced split count applied.
dash::BwdWorkspace bwd_workspace(const dash_problem* p) {
  dash::BwdWorkspace ws =
      dash::attn_bwd_tc_workspace(p->batch, p->n_q_heads, p->n_kv_heads, p->seq_len, n_chunks(p));
  if (g_bwd_split_forced > 0) {
    ws.n_split = g_bwd_split_forced;
    const size_t part = (size_t)ws.n_split * p->batch * p->n_kv_heads * p->seq_len * 256 * 4;
    ws.total = ws.p_off + (ws.n_split > 1 ? ((part + 255) & ~(size_t)255) : 0);
  }
  return ws;
}

size_t attn_bwd_ws_bytes(const dash_problem* p) {
  if (!attn_bwd_tc_applies(p)) return 0;
  return bwd_workspace(p).total;
}

template <int CHUNK>
int run_attn_bwd_tc(const dash_problem* p, const void* Q, const void* K, const void* V,
                    const float* w, const uint32_t* mask, const void* O, const float* lse,
                    const void* dO, float* dQ, float* dK, float* dV, float* dw, void* workspace,
                    cudaStream_t st) {
  constexpr uint64_t d = 128;
  const int G = p->n_q_heads / p->n_kv_heads;
  const int P = 128 / G;
  CUtensorMap tq, tdo, tk64, tv64, tk128, tv128;
  {
    // Q and dO viewed as (d, head, position): a box {64, G, P} lands
    // position-major, shared-memory row r = p * G + h
    const uint64_t dims[3] = {d, (uint64_t)p->batch * p->n_q_heads, (uint64_t)p->seq_len};
    const uint64_t str[2] = {(uint64_t)p->seq_len * d * 2, d * 2};
    const uint32_t box[3] = {64, (uint32_t)G, (uint32_t)P};
    if (!make_tmap(&tq, Q, 3, dims, str, box)) return DASH_ERR_CUDA;
    if (!make_tmap(&tdo, dO, 3, dims, str, box)) return DASH_ERR_CUDA;
  }
  {
    const uint64_t dims[2] = {d, (uint64_t)p->batch * p->n_kv_heads * p->seq_len};
    const uint64_t str[1] = {d * 2};
    const uint32_t box64[2] = {64, 64}, box128[2] = {64, 128};
    if (!make_tmap(&tk64, K, 2, dims, str, box64) || !make_tmap(&tv64, V, 2, dims, str, box64) ||
        !make_tmap(&tk128, K, 2, dims, str, box128) || !make_tmap(&tv128, V, 2, dims, str, box128))
      return DASH_ERR_CUDA;
  }
  dash::BwdParams prm;
  prm.w = w;
  prm.mask = mask;
  prm.lse = lse;
  prm.O = static_cast<const bf16*>(O);
  prm.dO = static_cast<const bf16*>(dO);
  prm.dQ = dQ;
  prm.dK = dK;
  prm.dV = dV;
  prm.dw = dw;
  prm.n_q = p->n_q_heads;
  prm.n_kv = p->n_kv_heads;
  prm.seq = p->seq_len;
  prm.chunk = p->chunk;
  prm.n_c = n_chunks(p);
  prm.nw = (prm.n_c + 31) / 32;
  prm.G = G;
  prm.lgG = G == 4 ? 2 : G == 8 ? 3 : 4;
  prm.P = P;
  prm.n_tiles = p->seq_len / P;
  prm.n_bg = p->batch * p->n_kv_heads;
  prm.sigma = p->sigma;
  prm.scale = 1.f / sqrtf((float)d);
  prm.scale_log2 = 1.4426950408889634f * prm.scale;
  const dash::BwdWorkspace ws = bwd_workspace(p);
  uint8_t* wsb = static_cast<uint8_t*>(workspace);
  prm.Drow = reinterpret_cast<float*>(wsb + ws.d_off);
  prm.tmask = reinterpret_cast<uint32_t*>(wsb + ws.t_off);
  prm.part = ws.n_split > 1 ? reinterpret_cast<float*>(wsb + ws.p_off) : nullptr;
  prm.n_split = ws.n_split;
  if (dw) {
    const cudaError_t e = cudaMemsetAsync(dw, 0, (size_t)prm.n_bg * p->seq_len * prm.n_c * sizeof(float), st);
    if (e != cudaSuccess) return cuda_status(e);
  }
  return cuda_status(dash::launch_attn_bwd_tc<CHUNK>(tq, tdo, tk64, tv64, tk128, tv128, prm, st));
}

}  // namespace

extern "C" {

const char* dash_status_str(int s) {
  switch (s) {
    case DASH_OK: return "DASH_OK";
    case DASH_ERR_INVALID_ARG: return "DASH_ERR_INVALID_ARG";
    case DASH_ERR_UNSUPPORTED: return "DASH_ERR_UNSUPPORTED";
    case DASH_ERR_CUDA: return "DASH_ERR_CUDA";
    case DASH_ERR_TIMEOUT: return "DASH_ERR_TIMEOUT";
    case DASH_ERR_WORKSPACE: return "DASH_ERR_WORKSPACE";
    default: return "DASH_ERR_UNKNOWN";
  }
}

int dash_version(void) { return (3 << 16) | 0; }

int dash_summarize(const dash_problem* p, const void* K, const float* qbar, int chunk_begin,
                   int chunk_end, void* Kbar, void* stream) {
  int rc = check_problem(p, true);
  if (rc) return rc;
  if (!K || !qbar || !Kbar || !aligned16(K) || !aligned16(qbar) || !aligned16(Kbar))
    return DASH_ERR_INVALID_ARG;
  const int full = p->seq_len / p->chunk;
  if (chunk_begin < 0 || chunk_end < chunk_begin || chunk_end > full) return DASH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (p->dtype == DASH_BF16) {
    e = p->head_dim == 128
            ? dash::launch_summarize<bf16, 128>(static_cast<const bf16*>(K), qbar, static_cast<bf16*>(Kbar),
                                                p->batch, p->n_kv_heads, p->seq_len, p->chunk, chunk_begin, chunk_end, st)
            : dash::launch_summarize<bf16, 64>(static_cast<const bf16*>(K), qbar, static_cast<bf16*>(Kbar),
                                               p->batch, p->n_kv_heads, p->seq_len, p->chunk, chunk_begin, chunk_end, st);
  } else {
    e = p->head_dim == 128
            ? dash::launch_summarize<float, 128>(static_cast<const float*>(K), qbar, static_cast<float*>(Kbar),
                                                 p->batch, p->n_kv_heads, p->seq_len, p->chunk, chunk_begin, chunk_end, st)
            : dash::launch_summarize<float, 64>(static_cast<const float*>(K), qbar, static_cast<float*>(Kbar),
                                                p->batch, p->n_kv_heads, p->seq_len, p->chunk, chunk_begin, chunk_end, st);
  }
  return cuda_status(e);
}

int dash_summarize_append(const dash_problem* p, const int32_t* cache_lens,
                          const int32_t* page_table, int max_pages, int n_pages, const void* K,
                          const float* qbar, void* Kbar, void* stream) {
  int rc = check_problem(p, true);
  if (rc) return rc;
  if (!K || !qbar || !Kbar || !aligned16(K) || !aligned16(qbar) || !aligned16(Kbar))
    return DASH_ERR_INVALID_ARG;
  if (!cache_lens || (reinterpret_cast<uintptr_t>(cache_lens) & 3u)) return DASH_ERR_INVALID_ARG;
  if (page_table && ((reinterpret_cast<uintptr_t>(page_table) & 3u) ||
                     max_pages < n_chunks(p) || n_pages < 1))
    return DASH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
#define DASH_APPEND(T, D)                                                                        \
  dash::launch_summarize_append<T, D>(static_cast<const T*>(K), qbar, static_cast<T*>(Kbar),     \
                                      cache_lens, page_table, max_pages, n_pages, p->batch,     \
                                      p->n_kv_heads, p->seq_len, p->chunk, st)
  if (p->dtype == DASH_BF16)
    e = p->head_dim == 128 ? DASH_APPEND(bf16, 128) : DASH_APPEND(bf16, 64);
  else
    e = p->head_dim == 128 ? DASH_APPEND(float, 128) : DASH_APPEND(float, 64);
#undef DASH_APPEND
  return cuda_status(e);
}

int dash_route_topk(const dash_problem* p, const void* Q, const void* Kbar, int k, float* w,
                    uint32_t* mask, void* stream) {
  int rc = check_problem(p, false);
  if (rc) return rc;
  if (!Q || !Kbar || !w || !mask || !aligned16(Q) || !aligned16(Kbar) || !aligned16(w) ||
      !aligned16(mask) || k < 1)
    return DASH_ERR_INVALID_ARG;
  if (n_chunks(p) > dash::kTopkMaxChunks || p->n_q_heads / p->n_kv_heads > 16) return DASH_ERR_UNSUPPORTED;
  if (p->estimate_diagonal) return DASH_ERR_UNSUPPORTED;   // no entmax normalisation to correct
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
#define DASH_TOPK(T, D)                                                                         \
  dash::launch_route_topk<T, D>(static_cast<const T*>(Q), static_cast<const T*>(Kbar), w, mask, \
                                p->batch, p->n_q_heads, p->n_kv_heads, p->seq_len, p->chunk, k,  \
                                p->gamma, st)
  if (p->dtype == DASH_BF16)
    e = p->head_dim == 128 ? DASH_TOPK(bf16, 128) : DASH_TOPK(bf16, 64);
  else
    e = p->head_dim == 128 ? DASH_TOPK(float, 128) : DASH_TOPK(float, 64);
#undef DASH_TOPK
  return cuda_status(e);
}

int dash_attn_bwd(const dash_problem* p, const void* Q, const void* K, const void* V,
                  const float* w, const uint32_t* mask, const void* O, const float* lse,
                  const void* dO, float* dQ, float* dK, float* dV, float* dw, void* workspace,
                  size_t workspace_bytes, void* stream) {
  int rc = check_problem(p, false);
  if (rc) return rc;
  const void* req[] = {Q, K, V, w, mask, O, lse, dO, dQ, dK, dV};
  for (const void* ptr : req)
    if (!ptr || !aligned16(ptr)) return DASH_ERR_INVALID_ARG;
  if (dw && !aligned16(dw)) return DASH_ERR_INVALID_ARG;
  if (p->n_q_heads / p->n_kv_heads > 16) return DASH_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (attn_bwd_tc_applies(p)) {
    const size_t need = attn_bwd_ws_bytes(p);
    if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
      return DASH_ERR_WORKSPACE;
    return p->chunk == 64
               ? run_attn_bwd_tc<64>(p, Q, K, V, w, mask, O, lse, dO, dQ, dK, dV, dw, workspace, st)
               : run_attn_bwd_tc<128>(p, Q, K, V, w, mask, O, lse, dO, dQ, dK, dV, dw, workspace, st);
  }
  const size_t kv_bytes = (size_t)p->batch * p->n_kv_heads * p->seq_len * p->head_dim * sizeof(float);
  cudaError_t e = cudaMemsetAsync(dK, 0, kv_bytes, st);
  if (e == cudaSuccess) e = cudaMemsetAsync(dV, 0, kv_bytes, st);
  if (e != cudaSuccess) return cuda_status(e);
#define DASH_BWD(T, D)                                                                          \
  dash::launch_attn_bwd<T, D>(static_cast<const T*>(Q), static_cast<const T*>(K),                \
                              static_cast<const T*>(V), w, mask, static_cast<const T*>(O), lse,  \
                              static_cast<const T*>(dO), dQ, dK, dV, dw, p->batch, p->n_q_heads, \
                              p->n_kv_heads, p->seq_len, p->chunk, p->sigma, st)
  if (p->dtype == DASH_BF16)
    e = p->head_dim == 128 ? DASH_BWD(bf16, 128) : DASH_BWD(bf16, 64);
  else
    e = p->head_dim == 128 ? DASH_BWD(float, 128) : DASH_BWD(float, 64);
#undef DASH_BWD
  return cuda_status(e);
}

int dash_route_bwd(const dash_problem* p, const void* Q, const void* Kbar, const float* dw,
                   float* dQ, float* dKbar, void* stream) {
  int rc = check_problem(p, false);
  if (rc) return rc;
  const void* req[] = {Q, Kbar, dw, dQ, dKbar};
  for (const void* ptr : req)
    if (!ptr || !aligned16(ptr)) return DASH_ERR_INVALID_ARG;
  if (p->n_q_heads / p->n_kv_heads > 16 || n_chunks(p) > dash::kRbMaxChunks) return DASH_ERR_UNSUPPORTED;
  if (p->estimate_diagonal) return DASH_ERR_UNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
#define DASH_RB(T, D)                                                                            \
  dash::launch_route_bwd<T, D>(static_cast<const T*>(Q), static_cast<const T*>(Kbar), dw, dQ,    \
                               dKbar, p->batch, p->n_q_heads, p->n_kv_heads, p->seq_len,         \
                               p->chunk, p->alpha, p->gamma, st)
  if (p->dtype == DASH_BF16)
    e = p->head_dim == 128 ? DASH_RB(bf16, 128) : DASH_RB(bf16, 64);
  else
    e = p->head_dim == 128 ? DASH_RB(float, 128) : DASH_RB(float, 64);
#undef DASH_RB
  return cuda_status(e);
}

int dash_summarize_bwd(const dash_problem* p, const void* K, const float* qbar, const float* dKbar,
                       float* dK, float* dqbar, void* stream) {
  int rc = check_problem(p, false);
  if (rc) return rc;
  const void* req[] = {K, qbar, dKbar, dK, dqbar};
  for (const void* ptr : req)
    if (!ptr || !aligned16(ptr)) return DASH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
#define DASH_SB(T, D)                                                                            \
  dash::launch_summarize_bwd<T, D>(static_cast<const T*>(K), qbar, dKbar, dK, dqbar, p->batch,  \
                                   p->n_kv_heads, p->seq_len, p->chunk, st)
  if (p->dtype == DASH_BF16)
    e = p->head_dim == 128 ? DASH_SB(bf16, 128) : DASH_SB(bf16, 64);
  else
    e = p->head_dim == 128 ? DASH_SB(float, 128) : DASH_SB(float, 64);
#undef DASH_SB
  return cuda_status(e);
}

}  // extern "C"

// dash_route (dense w) and dash_route_packed (compact weights, optional
// count / index)
static int route_entry(const dash_problem* p, const void* Q, const void* Kbar, const void* K,
                       const float* qbar, float* w, uint32_t* mask, bool packed, int32_t* count,
                       int32_t* index, void* stream) {
  int rc = check_problem(p, false);
  if (rc) return rc;
  if (!Q || !Kbar || !w || !mask || !aligned16(Q) || !aligned16(Kbar) || !aligned16(w) ||
      !aligned16(mask) || (count && !aligned16(count)) || (index && !aligned16(index)))
    return DASH_ERR_INVALID_ARG;
  if (p->estimate_diagonal && (!K || !qbar || !aligned16(K) || !aligned16(qbar)))
    return DASH_ERR_INVALID_ARG;
  if (n_chunks(p) > 2048) return DASH_ERR_UNSUPPORTED;
  if (!p->estimate_diagonal) {
    K = nullptr;
    qbar = nullptr;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
#define DASH_ROUTE(T, D)                                                                      \
  dash::launch_route<T, D>(static_cast<const T*>(Q), static_cast<const T*>(Kbar), w, mask,    \
                           static_cast<const T*>(K), qbar, p->batch, p->n_q_heads,            \
                           p->n_kv_heads, p->seq_len, p->chunk, p->alpha, p->gamma, st,       \
                           packed, count, index)
  const int G = p->n_q_heads / p->n_kv_heads;
  if (p->dtype == DASH_BF16 && p->head_dim == 128 && G == 16 && n_chunks(p) <= 1024)
    e = dash::launch_route_tc(static_cast<const bf16*>(Q), static_cast<const bf16*>(Kbar), w, mask,
                              static_cast<const bf16*>(K), qbar, p->batch, p->n_q_heads,
                              p->n_kv_heads, p->seq_len, p->chunk, p->alpha, p->gamma, st, packed,
                              count, index);
  else if (p->dtype == DASH_BF16)
    e = p->head_dim == 128 ? DASH_ROUTE(bf16, 128) : DASH_ROUTE(bf16, 64);
  else
    e = p->head_dim == 128 ? DASH_ROUTE(float, 128) : DASH_ROUTE(float, 64);
#undef DASH_ROUTE
  return cuda_status(e);
}

extern "C" {

int dash_route(const dash_problem* p, const void* Q, const void* Kbar, const void* K,
               const float* qbar, float* w, uint32_t* mask, void* stream) {
  return route_entry(p, Q, Kbar, K, qbar, w, mask, false, nullptr, nullptr, stream);
}

int dash_route_packed(const dash_problem* p, const void* Q, const void* Kbar, const void* K,
                      const float* qbar, uint32_t* mask, int32_t* count, int32_t* index,
                      float* weight, void* stream) {
  return route_entry(p, Q, Kbar, K, qbar, weight, mask, true, count, index, stream);
}

size_t dash_workspace_bytes(const dash_problem* p, int which) {
  if (which < 0 || which > 2) return 0;
  if (check_problem(p, which == 1) != DASH_OK) return 0;
  if (which == 0) return 0;
  if (which == 2) return attn_bwd_ws_bytes(p);
  return dash::decode_workspace_bytes(p->batch, p->n_q_heads, p->n_kv_heads, p->seq_len,
                                      p->head_dim, p->chunk);
}

}  // extern "C"

// dash_attn_fwd (dense w) and dash_attn_fwd_packed (compact weights)
static int attn_entry(const dash_problem* p, const void* Q, const void* K, const void* V,
                      const float* w, const uint32_t* mask, void* O, float* lse, bool packed,
                      void* stream) {
  int rc = check_problem(p, false);
  if (rc) return rc;
  if (!Q || !K || !V || !w || !mask || !O) return DASH_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(w) || !aligned16(mask) ||
      !aligned16(O) || (lse && !aligned16(lse)))
    return DASH_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p->dtype == DASH_F32) {
    cudaError_t e =
        p->head_dim == 128
            ? dash::launch_attn_f32<128>(static_cast<const float*>(Q), static_cast<const float*>(K),
                                         static_cast<const float*>(V), w, mask, static_cast<float*>(O), lse,
                                         p->batch, p->n_q_heads, p->n_kv_heads, p->seq_len, p->chunk, p->sigma,
                                         st, packed)
            : dash::launch_attn_f32<64>(static_cast<const float*>(Q), static_cast<const float*>(K),
                                        static_cast<const float*>(V), w, mask, static_cast<float*>(O), lse,
                                        p->batch, p->n_q_heads, p->n_kv_heads, p->seq_len, p->chunk, p->sigma,
                                        st, packed);
    return cuda_status(e);
  }
  const int G = p->n_q_heads / p->n_kv_heads;
  if (G != 4 && G != 8 && G != 16) return DASH_ERR_UNSUPPORTED;
  // a CTA covers 2 * 128 / G consecutive positions, all inside one chunk
  if (2 * (128 / G) > p->chunk || p->chunk % (2 * (128 / G)) != 0) return DASH_ERR_UNSUPPORTED;
  if (n_chunks(p) > 2048) return DASH_ERR_UNSUPPORTED;
  if (p->chunk == 64)
    return p->head_dim == 128 ? run_attn_tc<64, 128>(p, Q, K, V, w, mask, O, lse, packed, st)
                              : run_attn_tc<64, 64>(p, Q, K, V, w, mask, O, lse, packed, st);
  return p->head_dim == 128 ? run_attn_tc<128, 128>(p, Q, K, V, w, mask, O, lse, packed, st)
                            : run_attn_tc<128, 64>(p, Q, K, V, w, mask, O, lse, packed, st);
}

extern "C" {

int dash_attn_fwd(const dash_problem* p, const void* Q, const void* K, const void* V,
                  const float* w, const uint32_t* mask, void* O, float* lse, void* workspace,
                  size_t workspace_bytes, void* stream) {
  (void)workspace;
  (void)workspace_bytes;
  return attn_entry(p, Q, K, V, w, mask, O, lse, false, stream);
}

int dash_attn_fwd_packed(const dash_problem* p, const void* Q, const void* K, const void* V,
                         const float* weight, const uint32_t* mask, void* O, float* lse,
                         void* stream) {
  return attn_entry(p, Q, K, V, weight, mask, O, lse, true, stream);
}

// dash_decode, dash_decode_varlen (lens: nullable device [batch]) and
// dash_decode_paged (page_table: nullable device [batch][max_pages])
static int decode_entry(const dash_problem* p, const int32_t* lens, const int32_t* page_table,
                        int max_pages, int n_pages, const void* q,
                        const void* Kcache, const void* Vcache, const void* Kbar,
                        const float* qbar, void* o, float* lse, float* w, uint32_t* mask,
                        void* workspace, size_t workspace_bytes, void* stream) {
  int rc = check_problem(p, true);
  if (rc) return rc;
  if (!q || !Kcache || !Vcache || !Kbar || !o) return DASH_ERR_INVALID_ARG;
  if (p->estimate_diagonal && (!qbar || !aligned16(qbar))) return DASH_ERR_INVALID_ARG;
  if (!p->estimate_diagonal) qbar = nullptr;
  if (!aligned16(q) || !aligned16(Kcache) || !aligned16(Vcache) || !aligned16(Kbar) ||
      !aligned16(o) || (lse && !aligned16(lse)) || (w && !aligned16(w)) || (mask && !aligned16(mask)))
    return DASH_ERR_INVALID_ARG;
  if (p->dtype != DASH_BF16) return DASH_ERR_UNSUPPORTED;
  const int G = p->n_q_heads / p->n_kv_heads;
  if (G > 16 || n_chunks(p) > 2048 || p->batch * p->n_kv_heads > 64) return DASH_ERR_UNSUPPORTED;
  const size_t need = dash::decode_workspace_bytes(p->batch, p->n_q_heads, p->n_kv_heads,
                                                   p->seq_len, p->head_dim, p->chunk);
  if (!workspace || workspace_bytes < need || (reinterpret_cast<uintptr_t>(workspace) & 255u))
    return DASH_ERR_WORKSPACE;
  rc = dash::run_decode(p->batch, p->n_q_heads, p->n_kv_heads, p->seq_len, p->head_dim,
                        p->chunk, p->alpha, p->gamma, p->sigma, lens, page_table, max_pages,
                        n_pages, static_cast<const bf16*>(q),
                        static_cast<const bf16*>(Kcache), static_cast<const bf16*>(Vcache),
                        static_cast<const bf16*>(Kbar), qbar, static_cast<bf16*>(o), lse, w,
                        mask, workspace, static_cast<cudaStream_t>(stream));
  if (rc == DASH_ERR_CUDA) (void)cudaGetLastError();
  return rc;
}

int dash_decode(const dash_problem* p, const void* q, const void* Kcache, const void* Vcache,
                const void* Kbar, const float* qbar, void* o, float* lse, float* w,
                uint32_t* mask, void* workspace, size_t workspace_bytes, void* stream) {
  return decode_entry(p, nullptr, nullptr, 0, 0, q, Kcache, Vcache, Kbar, qbar, o, lse, w, mask,
                      workspace, workspace_bytes, stream);
}

int dash_decode_varlen(const dash_problem* p, const int32_t* cache_lens, const void* q,
                       const void* Kcache, const void* Vcache, const void* Kbar,
                       const float* qbar, void* o, float* lse, float* w, uint32_t* mask,
                       void* workspace, size_t workspace_bytes, void* stream) {
  if (!cache_lens || (reinterpret_cast<uintptr_t>(cache_lens) & 3u)) return DASH_ERR_INVALID_ARG;
  return decode_entry(p, cache_lens, nullptr, 0, 0, q, Kcache, Vcache, Kbar, qbar, o, lse, w,
                      mask, workspace, workspace_bytes, stream);
}

int dash_decode_paged(const dash_problem* p, const int32_t* cache_lens, const int32_t* page_table,
                      int max_pages, int n_pages, const void* q, const void* Kpool,
                      const void* Vpool, const void* Kbar, const float* qbar, void* o, float* lse,
                      float* w, uint32_t* mask, void* workspace, size_t workspace_bytes,
                      void* stream) {
  int rc = check_problem(p, true);
  if (rc) return rc;
  if (!cache_lens || (reinterpret_cast<uintptr_t>(cache_lens) & 3u) || !page_table ||
      (reinterpret_cast<uintptr_t>(page_table) & 3u))
    return DASH_ERR_INVALID_ARG;
  if (max_pages < n_chunks(p) || n_pages < 1) return DASH_ERR_INVALID_ARG;
  // TMA row coordinates are 32-bit
  if ((long long)n_pages * p->n_kv_heads * p->chunk > 0x7fffffffLL) return DASH_ERR_UNSUPPORTED;
  return decode_entry(p, cache_lens, page_table, max_pages, n_pages, q, Kpool, Vpool, Kbar, qbar,
                      o, lse, w, mask, workspace, workspace_bytes, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// dash_decode_noalloc: dash_decode with its scratch in a fixed device array.
//
// For callers that must not allocate device memory themselves: an engine
// that owns every byte of the GPU through its own pool, or a plugin API that
// forbids allocation.  The decode scratch (routing scores, active-chunk
// lists, split-KV partials) lives in the static array below, reserved on
// every GPU that loads this library until the process exits.
// ---------------------------------------------------------------------------
namespace dash {

// Failure-path self-test: one bounded wait on an mbarrier that nothing ever
// completes.  It runs out after the library's wait limit, records the
// timeout in the device error word exactly as a stalled kernel would, and
// returns; nothing faults, traps or hangs.
__global__ void selftest_wait_kernel() {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) (void)mbar_wait(&bar, 0, nullptr);
}

// Evaluates the attention kernel's FMA-pipe 2^x (exp2_poly2) on n inputs, so
// that its error can be measured against 2^x itself.
__global__ void selftest_exp2_poly_kernel(const float* __restrict__ x, float* __restrict__ y, int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x1 = i + 1 < n ? x[i + 1] : 0.f;
  float e0, e1;
  exp2_poly2(f2_pack(x[i], x1), e0, e1);
  y[i] = e0;
  if (i + 1 < n) y[i + 1] = e1;
}

}  // namespace dash

namespace {

constexpr size_t kDecodeStaticScratchBytes = size_t(8) << 20;   // 8 MiB
static __device__ __align__(256) uint8_t g_decode_static_scratch[kDecodeStaticScratchBytes];

// Device address of the static scratch on the current device.  In host code
// the array's name is only a stand-in, so the address is looked up with the
// device current.  The lookup is repeated on every call (after the first call
// on a device has loaded the library's device code it is a table lookup), so
// a device reset or a re-created primary context never leaves a stale
// address behind.
int static_scratch(void** out) {
  void* ptr = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&ptr, g_decode_static_scratch);
  if (e != cudaSuccess || !ptr) return cuda_status(e == cudaSuccess ? cudaErrorUnknown : e);
  *out = ptr;
  return DASH_OK;
}

}  // namespace

extern "C" {

int dash_decode_noalloc(const dash_problem* p, const void* q, const void* Kcache,
                        const void* Vcache, const void* Kbar, void* o, float* lse, float* w,
                        uint32_t* mask, void* stream) {
  int rc = check_problem(p, true);
  if (rc) return rc;
  if (!q || !Kcache || !Vcache || !Kbar || !o) return DASH_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(Kcache) || !aligned16(Vcache) || !aligned16(Kbar) ||
      !aligned16(o) || (lse && !aligned16(lse)) || (w && !aligned16(w)) || (mask && !aligned16(mask)))
    return DASH_ERR_INVALID_ARG;
  if (p->dtype != DASH_BF16 || p->estimate_diagonal) return DASH_ERR_UNSUPPORTED;
  const int G = p->n_q_heads / p->n_kv_heads;
  if (G > 16 || n_chunks(p) > 2048 || p->batch * p->n_kv_heads > 64) return DASH_ERR_UNSUPPORTED;
  const size_t need = dash::decode_workspace_bytes(p->batch, p->n_q_heads, p->n_kv_heads,
                                                   p->seq_len, p->head_dim, p->chunk);
  if (need > kDecodeStaticScratchBytes) return DASH_ERR_WORKSPACE;
  void* scratch = nullptr;
  rc = static_scratch(&scratch);
  if (rc) return rc;
  // Nothing in the scratch has to start at zero: every element the decode
  // kernels read is written earlier in the same call.
  rc = dash::run_decode(p->batch, p->n_q_heads, p->n_kv_heads, p->seq_len, p->head_dim,
                        p->chunk, p->alpha, p->gamma, p->sigma, nullptr, nullptr, 0, 0,
                        static_cast<const bf16*>(q),
                        static_cast<const bf16*>(Kcache), static_cast<const bf16*>(Vcache),
                        static_cast<const bf16*>(Kbar), nullptr, static_cast<bf16*>(o), lse, w,
                        mask, scratch, static_cast<cudaStream_t>(stream));
  if (rc == DASH_ERR_CUDA) (void)cudaGetLastError();
  return rc;
}

int dash_selftest_wait_timeout(void* stream) {
  dash::selftest_wait_kernel<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>();
  return cuda_status(cudaGetLastError());
}

int dash_selftest_bwd_split(int n) {
  if (n < 0 || n > dash::kBwdMaxSplit) return -1;
  const int prev = g_bwd_split_forced;
  g_bwd_split_forced = n;
  return prev;
}

int dash_selftest_exp2_poly(const float* x, float* y, int n, void* stream) {
  if (n < 0 || (n > 0 && (!x || !y))) return DASH_ERR_INVALID_ARG;
  if (n == 0) return DASH_OK;
  const int pairs = (n + 1) / 2;
  dash::selftest_exp2_poly_kernel<<<(pairs + 255) / 256, 256, 0, static_cast<cudaStream_t>(stream)>>>(x, y, n);
  return cuda_status(cudaGetLastError());
}

int dash_get_error(void* stream) {
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return DASH_ERR_CUDA;
  unsigned int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, dash::g_dash_error, sizeof(v)) != cudaSuccess) return DASH_ERR_CUDA;
  if (v && cudaMemcpyToSymbol(dash::g_dash_error, &zero, sizeof(zero)) != cudaSuccess)
    return DASH_ERR_CUDA;
  if (v & dash::DASH_DEV_ERR_TIMEOUT) return DASH_ERR_TIMEOUT;
  if (v & dash::DASH_DEV_ERR_ARG) return DASH_ERR_INVALID_ARG;
  return v ? DASH_ERR_UNSUPPORTED : DASH_OK;
}

}  // extern "C"
