// Stage 2 (fp32): prior-induced block-sparse softmax attention on CUDA cores.
//
// Same operation as the tcgen05 kernel (gist.science technical summary,
// "Fase 2"): bias 0 on the query's own chunk (causal), sigma * ln w on an
// active routed chunk, -inf elsewhere; online softmax over the keys.  fp32
// inputs want fp32 products, which the tensor cores do not give, so this
// path uses one warp per (b, query head, position), lanes split over the
// head dimension.  It serves the small fp32 workload.
#pragma once

#include "dash_common.cuh"

namespace dash {

// PACKED: w is the compact form of stage 1 (per row, the weights of the
// routed chunks in increasing chunk order), else dense [rows][n_c].
template <int D, bool PACKED>
__global__ void __launch_bounds__(256) attn_f32_kernel(
    const float* __restrict__ Q, const float* __restrict__ K, const float* __restrict__ V,
    const float* __restrict__ w, const uint32_t* __restrict__ mask, float* __restrict__ O,
    float* __restrict__ lse, int n_q, int n_kv, int seq, int chunk, int n_c, float sigma,
    float scale_log2, long long n_rows) {
  constexpr int CPL = D / 32;                    // columns per lane
  const long long row = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (row >= n_rows) return;
  const int i = (int)(row % seq);
  const long long bh = row / seq;                // b * n_q + h
  const int h = (int)(bh % n_q);
  const int b = (int)(bh / n_q);
  const int G = n_q / n_kv;
  const int g = h / G;
  const int c_i = i / chunk;
  const int nw = (n_c + 31) >> 5;
  const size_t bg = (size_t)b * n_kv + g;
  const float* Kb = K + bg * seq * D;
  const float* Vb = V + bg * seq * D;
  const float* wrow = w + (bg * seq + i) * n_c;
  const uint32_t* mrow = mask + (bg * seq + i) * nw;

  float q[CPL], acc[CPL];
#pragma unroll
  for (int e = 0; e < CPL; ++e) {
    q[e] = Q[row * D + lane + 32 * e] * scale_log2;
    acc[e] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  auto visit = [&](int j, float bias) {
    float part = 0.f;
#pragma unroll
    for (int e = 0; e < CPL; ++e) part = fmaf(q[e], Kb[(size_t)j * D + lane + 32 * e], part);
    const float s = warp_sum(part) + bias;
    const float m_new = fmaxf(m, s);
    const float corr = exp2f(m - m_new);
    const float pj = exp2f(s - m_new);
    l = l * corr + pj;
#pragma unroll
    for (int e = 0; e < CPL; ++e) acc[e] = fmaf(pj, Vb[(size_t)j * D + lane + 32 * e], acc[e] * corr);
    m = m_new;
  };
  for (int j = c_i * chunk; j <= i; ++j) visit(j, 0.f);          // diagonal branch first
  int rank = 0;                                                   // routed chunks seen so far
  for (int c = 0; c < c_i && c < n_c; ++c) {
    if (!((mrow[c >> 5] >> (c & 31)) & 1u)) continue;
    const float wc = PACKED ? wrow[rank++] : wrow[c];
    const float bias = sigma == 0.f ? 0.f : sigma * log2f(wc);
    if (bias == -INFINITY) continue;
    for (int j = c * chunk; j < (c + 1) * chunk; ++j) visit(j, bias);
  }
  const float inv = 1.f / l;
#pragma unroll
  for (int e = 0; e < CPL; ++e) O[row * D + lane + 32 * e] = acc[e] * inv;
  if (lse && lane == 0) lse[row] = (m + log2f(l)) * 0.69314718055994531f;
}

template <int D>
cudaError_t launch_attn_f32(const float* Q, const float* K, const float* V, const float* w,
                            const uint32_t* mask, float* O, float* lse, int batch, int n_q,
                            int n_kv, int seq, int chunk, float sigma, cudaStream_t st,
                            bool packed = false) {
  const int n_c = (seq + chunk - 1) / chunk;
  const long long n_rows = (long long)batch * n_q * seq;
  const int threads = 256;
  const long long blocks = (n_rows * 32 + threads - 1) / threads;
  const float scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  if (packed)
    attn_f32_kernel<D, true><<<(unsigned)blocks, threads, 0, st>>>(
        Q, K, V, w, mask, O, lse, n_q, n_kv, seq, chunk, n_c, sigma, scale_log2, n_rows);
  else
    attn_f32_kernel<D, false><<<(unsigned)blocks, threads, 0, st>>>(
        Q, K, V, w, mask, O, lse, n_q, n_kv, seq, chunk, n_c, sigma, scale_log2, n_rows);
  return cudaGetLastError();
}

}  // namespace dash
