// Stage 0: chunk summary by learned-query local SDPA.
//
// gist.science technical summary, "Fase 0: Lokale Chunk Samenvatting": a
// learned query q_bar attends to the B keys of each chunk with scaled
// dot-product attention; the summary is the attention-weighted mean of the
// keys (q_bar = 0 gives mean pooling).
//
// One warp per (b, h_kv, chunk), single pass over the chunk with an online
// softmax.  The chunk (B rows of d elements, contiguous in memory) is read
// with coalesced 16-byte loads: each row is split over LPR = d*sizeof(T)/16
// lanes, and a warp reads RPW = 32/LPR rows per step.  HBM-bound: K is read
// once, the summaries are B times smaller.
#pragma once

#include "dash_common.cuh"

namespace dash {

// One warp: the summary of the `chunk` rows at `base` (rows of D elements,
// contiguous) with the learned query qh (D floats), written to dst (D elements
// of OutT: the keys' type for the summary cache, float for the estimated
// summary of a partial chunk that routing uses without storing it).
// UNROLL row groups are loaded per round; the rows are processed in the same
// order whatever UNROLL is, so the result does not depend on it.
template <typename T, int D, int UNROLL, typename OutT = T>
__device__ __forceinline__ void summarize_chunk_warp(const T* __restrict__ base,
                                                     const float* __restrict__ qh,
                                                     OutT* __restrict__ dst, int chunk, int lane) {
  constexpr int EPV = 16 / sizeof(T);      // elements per 16-byte vector
  constexpr int LPR = D / EPV;             // lanes per row
  constexpr int RPW = 32 / LPR;            // rows per warp step
  static_assert(LPR >= 1 && LPR <= 32 && (32 % LPR) == 0, "bad row split");

  const int sub = lane % LPR;                   // which 16-byte column group
  const int grp = lane / LPR;                   // which row of the step
  float q[EPV];
  const float rs = rsqrtf((float)D);
#pragma unroll
  for (int e = 0; e < EPV; ++e) q[e] = qh[sub * EPV + e] * rs;

  float m = -INFINITY, l = 0.f;
  float acc[EPV];
#pragma unroll
  for (int e = 0; e < EPV; ++e) acc[e] = 0.f;

  for (int r0 = 0; r0 < chunk; r0 += RPW * UNROLL) {
    uint4 raw[UNROLL];
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int row = r0 + u * RPW + grp;
      raw[u] = row < chunk ? __ldg(reinterpret_cast<const uint4*>(base + (size_t)row * D) + sub)
                           : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < UNROLL; ++u) {
      const int row0 = r0 + u * RPW;
      if (row0 >= chunk) break;
      const T* v = reinterpret_cast<const T*>(&raw[u]);
      float x[EPV];
      float part = 0.f;
#pragma unroll
      for (int e = 0; e < EPV; ++e) {
        x[e] = Elem<T>::to_f(v[e]);
        part = fmaf(q[e], x[e], part);
      }
#pragma unroll
      for (int o = LPR / 2; o > 0; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
      // every lane now holds the score of its own row; gather all RPW scores
      // (rows past `chunk` -- a partial last group, when the rows are the
      // visible part of a chunk -- take no part: score -inf)
      float s[RPW];
      float smax = -INFINITY;
#pragma unroll
      for (int r = 0; r < RPW; ++r) {
        const float sr = __shfl_sync(0xffffffffu, part, r * LPR);
        s[r] = row0 + r < chunk ? sr : -INFINITY;
        smax = fmaxf(smax, s[r]);
      }
      const float m_new = fmaxf(m, smax);
      const float corr = __expf(m - m_new);
      float psum = 0.f;
#pragma unroll
      for (int r = 0; r < RPW; ++r) psum += __expf(s[r] - m_new);
      const float pown = __expf((row0 + grp < chunk ? part : -INFINITY) - m_new);
      l = l * corr + psum;
#pragma unroll
      for (int e = 0; e < EPV; ++e) acc[e] = fmaf(pown, x[e], acc[e] * corr);
      m = m_new;
    }
  }
  // lanes with the same `sub` hold partial sums over disjoint rows
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < EPV; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], o);
  if (grp == 0) {
    const float inv = 1.f / l;
    if constexpr (sizeof(OutT) == sizeof(T)) {
      OutT outv[EPV];
#pragma unroll
      for (int e = 0; e < EPV; ++e) outv[e] = Elem<OutT>::from_f(acc[e] * inv);
      *reinterpret_cast<uint4*>(dst + sub * EPV) = *reinterpret_cast<const uint4*>(outv);
    } else {
#pragma unroll
      for (int e = 0; e < EPV; ++e) dst[sub * EPV + e] = Elem<OutT>::from_f(acc[e] * inv);
    }
  }
}

template <typename T, int D>
__global__ void __launch_bounds__(256) summarize_kernel(
    const T* __restrict__ K, const float* __restrict__ qbar, T* __restrict__ Kbar,
    int n_kv, int seq, int chunk, int chunk_begin, int n_chunks_out, int kbar_rows,
    int n_warps_total) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= n_warps_total) return;
  const int c_local = warp % n_chunks_out;
  const int bh = warp / n_chunks_out;           // b * n_kv + h
  const int h = bh % n_kv;
  const int c = chunk_begin + c_local;
  // many warps in flight: four row groups per round suffice
  summarize_chunk_warp<T, D, 4>(K + ((size_t)bh * seq + (size_t)c * chunk) * D, qbar + h * D,
                                Kbar + ((size_t)bh * kbar_rows + c) * D, chunk, lane);
}

// Summary-cache append for incremental decoding with a length per sequence:
// one warp per (b, h_kv); a sequence whose length L_b is a multiple of the
// chunk size has just completed chunk L_b / B - 1, whose summary is written
// (the same arithmetic as summarize_kernel, so the same bits).  K is the
// cache [b][n_kv][L][D], or with page_table the page pool [n_pages][n_kv][B][D].
template <typename T, int D>
__global__ void __launch_bounds__(256) summarize_append_kernel(
    const T* __restrict__ K, const float* __restrict__ qbar, T* __restrict__ Kbar,
    const int* __restrict__ lens, const int* __restrict__ page_table, int max_pages, int n_pages,
    int batch, int n_kv, int L, int chunk) {
  const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (warp >= batch * n_kv) return;
  const int b = warp / n_kv, h = warp % n_kv;
  const int Lb = __ldg(lens + b);
  if (Lb < 1 || Lb > L) {
    if (lane == 0 && h == 0) atomicOr(&g_dash_error, DASH_DEV_ERR_ARG);
    return;
  }
  if (Lb % chunk != 0) return;                  // no chunk completed at this length
  const int c = Lb / chunk - 1;
  const T* base;
  if (page_table) {
    const int pg = __ldg(page_table + (size_t)b * max_pages + c);
    if (pg < 0 || pg >= n_pages) {
      if (lane == 0) atomicOr(&g_dash_error, DASH_DEV_ERR_ARG);
      return;
    }
    base = K + ((size_t)pg * n_kv + h) * chunk * D;
  } else {
    base = K + ((size_t)warp * L + (size_t)c * chunk) * D;
  }
  // one warp per sequence and head, so few in flight: a 64-row chunk is
  // loaded in one round (two for 128 rows)
  summarize_chunk_warp<T, D, 32>(base, qbar + h * D, Kbar + ((size_t)warp * (L / chunk) + c) * D,
                                 chunk, lane);
}

template <typename T, int D>
cudaError_t launch_summarize(const T* K, const float* qbar, T* Kbar, int batch, int n_kv, int seq,
                             int chunk, int chunk_begin, int chunk_end, cudaStream_t st) {
  const int n_out = chunk_end - chunk_begin;
  if (n_out <= 0) return cudaSuccess;
  const int warps = batch * n_kv * n_out;
  const int threads = 256;
  const int blocks = (warps * 32 + threads - 1) / threads;
  summarize_kernel<T, D><<<blocks, threads, 0, st>>>(K, qbar, Kbar, n_kv, seq, chunk, chunk_begin,
                                                    n_out, seq / chunk, warps);
  return cudaGetLastError();
}

template <typename T, int D>
cudaError_t launch_summarize_append(const T* K, const float* qbar, T* Kbar, const int* lens,
                                    const int* page_table, int max_pages, int n_pages, int batch,
                                    int n_kv, int L, int chunk, cudaStream_t st) {
  const int warps = batch * n_kv;
  const int threads = 256;
  const int blocks = (warps * 32 + threads - 1) / threads;
  summarize_append_kernel<T, D><<<blocks, threads, 0, st>>>(K, qbar, Kbar, lens, page_table,
                                                           max_pages, n_pages, batch, n_kv, L, chunk);
  return cudaGetLastError();
}

}  // namespace dash
