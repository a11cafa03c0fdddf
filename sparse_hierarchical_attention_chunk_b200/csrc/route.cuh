// Stage 1: alpha-entmax chunk routing with GQA averaging and a bit-packed mask.
//
// gist.science technical summary, "Fase 1: Entmax Chunk Routering": per
// query, logits z_bar against the chunk summaries, w_hat = alpha-entmax(gamma
// z_bar) (support set by a score-dependent threshold tau, aiexpert.news method
// paragraph), and, under GQA, the probabilities of the query heads sharing a
// KV head are averaged so the group shares one support.
//
// Work decomposition.  One CTA (8 warps) owns 8 consecutive query positions
// of one (b, h_kv); they lie in one chunk and share the eligible set
// c < c_i.  The G query heads are processed two at a time: a pass computes
// the 16 x n_elig logit tile (2 heads x 8 positions) into shared memory
// (bf16: mma.sync m16n8k16 with fp32 accumulation, K-bar fragments read
// straight from L2; fp32: CUDA-core FMAs), then warp p runs the entmax of
// its position's two rows.  Each lane keeps NV = n_c/32 values of a row in
// registers; tau is the root of f(tau) = sum_c [x_c - tau]_+^e - 1
// (e = 1/(alpha-1)).  It is found by Newton's method from tau = max x - 1 on
// h(tau) = ||[x - tau]_+||_e - 1, which has the same root, is convex and
// decreasing (so the iterates rise monotonically to the root) and is nearly
// linear (so few steps are needed); for alpha = 1.5 a final exact step solves
// the quadratic on the support found.  The GQA mean stays
// in registers across passes; the mask word is a warp ballot of w > 0.
#pragma once

#include "dash_common.cuh"
#include "summarize.cuh"

namespace dash {

enum EntmaxKind { kEntmax15 = 0, kSparsemax = 1, kEntmaxGeneric = 2 };

template <int KIND>
__device__ __forceinline__ float entmax_pow(float d, float e) {   // d >= 0
  if (KIND == kEntmax15) return d * d;
  if (KIND == kSparsemax) return d;
  return d > 0.f ? ex2f(e * lg2f(d)) : 0.f;
}

// Threshold tau of alpha-entmax for the NV values x held by each lane of a
// warp (x = (alpha-1) gamma z; -inf marks an ineligible entry).  At least
// one entry must be finite.  Warp-uniform result.
template <int NV, int KIND>
__device__ __forceinline__ float entmax_tau_warp(const float (&x)[NV], float e) {
  float m = -INFINITY;
#pragma unroll
  for (int k = 0; k < NV; ++k) m = fmaxf(m, x[k]);
  m = warp_max(m);
  float tau = m - 1.f;                       // f(tau) >= 0 here
  for (int it = 0; it < 48; ++it) {
    float s0 = 0.f, s1 = 0.f;                // s0 = sum d^e, s1 = sum d^(e-1) (times e)
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const float d = fmaxf(x[k] - tau, 0.f);
      if (KIND == kEntmax15) {
        s0 = fmaf(d, d, s0);
        s1 += d;
      } else if (KIND == kSparsemax) {
        s0 += d;
        s1 += d > 0.f ? 1.f : 0.f;
      } else {
        const float pe = entmax_pow<KIND>(d, e);
        s0 += pe;
        s1 += d > 0.f ? pe / d : 0.f;
      }
    }
    s0 = warp_sum(s0);
    s1 = warp_sum(s1);
    const float f = s0 - 1.f;
    if (!(f > 0.f) || !(s1 > 0.f)) break;
    // Newton on h(tau) = ||[x - tau]_+||_e - 1 (e-norm, e = 1/(alpha-1) >= 1):
    // convex and decreasing like f but almost linear, so far fewer steps.
    //   h = N - 1, h' = -N^(1-e) sum d^(e-1), N = (sum d^e)^(1/e)
    float step;
    if (KIND == kEntmax15) {
      const float nrm = sqrtf(s0);                // s1 = sum d
      step = (s0 - nrm) / s1;
    } else if (KIND == kSparsemax) {
      step = f / s1;                              // h = f, s1 = support size
    } else {
      const float nrm = ex2f(lg2f(s0) / e);       // s1 = sum d^(e-1)
      step = (nrm - 1.f) * s0 / (nrm * s1);       // (N - 1) N^(e-1) / sum d^(e-1)
    }
    const float nt = tau + step;
    if (!(nt > tau)) break;                  // no further progress in fp32
    tau = nt;
    if (f < 1e-6f) break;
  }
  if (KIND == kEntmax15) {
    // exact root of sum_{S} (x - tau')^2 = 1 on the current support S, taken
    // relative to tau so that no large numbers cancel:
    // delta = (D2 - 1) / (D1 + sqrt(D1^2 - k (D2 - 1)))
    float d1 = 0.f, d2 = 0.f, kk = 0.f;
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const float d = x[k] - tau;
      if (d > 0.f) { d1 += d; d2 = fmaf(d, d, d2); kk += 1.f; }
    }
    d1 = warp_sum(d1);
    d2 = warp_sum(d2);
    kk = warp_sum(kk);
    const float disc = d1 * d1 - kk * (d2 - 1.f);
    if (kk > 0.f && disc >= 0.f) {
      const float delta = (d2 - 1.f) / (d1 + sqrtf(disc));
      const float tc = tau + delta;
      // accept only if every element of S stays above the new threshold
      bool ok = true;
#pragma unroll
      for (int k = 0; k < NV; ++k)
        if (x[k] > tau && !(x[k] > tc)) ok = false;
      if (__all_sync(0xffffffffu, ok)) tau = tc;
    }
  } else if (KIND == kSparsemax) {
    float d1 = 0.f, kk = 0.f;
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const float d = x[k] - tau;
      if (d > 0.f) { d1 += d; kk += 1.f; }
    }
    d1 = warp_sum(d1);
    kk = warp_sum(kk);
    if (kk > 0.f) {
      const float tc = tau + (d1 - 1.f) / kk;
      bool ok = true;
#pragma unroll
      for (int k = 0; k < NV; ++k)
        if (x[k] > tau && !(x[k] > tc)) ok = false;
      if (__all_sync(0xffffffffu, ok)) tau = tc;
    }
  }
  return tau;
}

__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], const uint32_t (&a)[4],
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// 16 x n_elig logits (rows: hsel * 8 + p, p < 8) into Ls[row * LS + c].
template <typename T, int D>
struct RouteLogits;

template <int D>
struct RouteLogits<__nv_bfloat16, D> {
  static __device__ __forceinline__ void run(const __nv_bfloat16* __restrict__ Q,
                                             const __nv_bfloat16* __restrict__ Kb, float* Ls,
                                             int LS, int n_elig, size_t qrow0, size_t qrow1,
                                             bool row1_valid) {
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, t = lane & 3;
    constexpr int KS = D / 16;
    uint32_t a[KS][4];
    const uint32_t* q0 = reinterpret_cast<const uint32_t*>(Q + qrow0 + (size_t)g * D);
    const uint32_t* q1 = reinterpret_cast<const uint32_t*>(Q + qrow1 + (size_t)g * D);
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      a[kk][0] = __ldg(q0 + kk * 8 + t);
      a[kk][1] = row1_valid ? __ldg(q1 + kk * 8 + t) : 0u;
      a[kk][2] = __ldg(q0 + kk * 8 + t + 4);
      a[kk][3] = row1_valid ? __ldg(q1 + kk * 8 + t + 4) : 0u;
    }
    const int n_tiles = (n_elig + 7) >> 3;
    for (int nt = warp; nt < n_tiles; nt += 8) {
      const int cc = nt * 8 + g;
      uint32_t b[KS][2];
      const uint32_t* kr = reinterpret_cast<const uint32_t*>(Kb + (size_t)cc * D);
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        b[kk][0] = cc < n_elig ? __ldg(kr + kk * 8 + t) : 0u;
        b[kk][1] = cc < n_elig ? __ldg(kr + kk * 8 + t + 4) : 0u;
      }
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) mma_bf16_16816(acc, a[kk], b[kk][0], b[kk][1]);
      const int col = nt * 8 + 2 * t;
      *reinterpret_cast<float2*>(Ls + g * LS + col) = make_float2(acc[0], acc[1]);
      *reinterpret_cast<float2*>(Ls + (g + 8) * LS + col) = make_float2(acc[2], acc[3]);
    }
  }
};

template <int D>
struct RouteLogits<float, D> {
  static __device__ __forceinline__ void run(const float* __restrict__ Q,
                                             const float* __restrict__ Kb, float* Ls, int LS,
                                             int n_elig, size_t qrow0, size_t qrow1,
                                             bool row1_valid) {
    for (int idx = threadIdx.x; idx < 16 * n_elig; idx += blockDim.x) {
      const int r = idx / n_elig, c = idx % n_elig;
      const int hsel = r >> 3, p = r & 7;
      float acc = 0.f;
      if (hsel == 0 || row1_valid) {
        const float* q = Q + (hsel ? qrow1 : qrow0) + (size_t)p * D;
        const float* k = Kb + (size_t)c * D;
#pragma unroll 8
        for (int j = 0; j < D; ++j) acc = fmaf(q[j], k[j], acc);
      }
      Ls[r * LS + c] = acc;
    }
  }
};

// estimate_diagonal (K, qbar non-null): the query's own chunk c_i joins each
// head's entmax as one more candidate; its logit is q . (stage 0's summary of
// the keys c_i B .. i), its group-mean weight goes to w[c_i] and it never
// sets a mask bit.
template <typename T, int D, int NV, int KIND>
__global__ void __launch_bounds__(256) route_kernel(
    const T* __restrict__ Q, const T* __restrict__ Kbar, float* __restrict__ w,
    uint32_t* __restrict__ mask, const T* __restrict__ K, const float* __restrict__ qbar,
    int32_t* __restrict__ count, int32_t* __restrict__ index, int packed, int n_q, int n_kv,
    int seq, int chunk, int n_c, int kbar_rows, float xscale, float e, int n_bg) {
  extern __shared__ __align__(16) float Ls[];
  __shared__ float khat[8][D];                 // estimate_diagonal: summary per position
  const int G = n_q / n_kv;
  const int n_tiles = seq >> 3;
  const int tile = n_tiles - 1 - (int)(blockIdx.x / n_bg);   // heavy (late) tiles first
  const int bg = blockIdx.x % n_bg;
  const int b = bg / n_kv, g = bg % n_kv;
  const int pos0 = tile * 8;
  const int c_i = pos0 / chunk;
  const int n_elig = min(c_i, n_c);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int LS = ((n_elig + 7) & ~7) + 4;
  const T* Kb = Kbar + (size_t)bg * kbar_rows * D;

  float wacc[NV];
#pragma unroll
  for (int k = 0; k < NV; ++k) wacc[k] = 0.f;

  const bool diag = K != nullptr;
  const bool dg = diag && n_elig > 0;
  if (dg) {
    // warp p: the visible keys of position pos0 + p in its own chunk
    summarize_chunk_warp<T, D, 4, float>(K + ((size_t)bg * seq + (size_t)c_i * chunk) * D,
                                         qbar + g * D, khat[warp], pos0 + warp - c_i * chunk + 1,
                                         lane);
    __syncwarp();
  }
  if (n_elig > 0) {
    for (int h0 = 0; h0 < G; h0 += 2) {
      const bool row1_valid = h0 + 1 < G;
      const size_t qrow0 = (((size_t)b * n_q + g * G + h0) * seq + pos0) * D;
      const size_t qrow1 = row1_valid ? qrow0 + (size_t)seq * D : qrow0;
      RouteLogits<T, D>::run(Q, Kb, Ls, LS, n_elig, qrow0, qrow1, row1_valid);
      __syncthreads();
#pragma unroll 1
      for (int hsel = 0; hsel < 2; ++hsel) {
        if (hsel == 1 && !row1_valid) break;
        const float* row = Ls + (hsel * 8 + warp) * LS;
        float xd = -INFINITY;
        if (dg) {
          const T* qr = Q + (hsel ? qrow1 : qrow0) + (size_t)warp * D;
          float acc = 0.f;
          for (int j = lane; j < D; j += 32) acc = fmaf(Elem<T>::to_f(qr[j]), khat[warp][j], acc);
          xd = xscale * warp_sum(acc);
        }
        float x[NV];
#pragma unroll
        for (int k = 0; k < NV; ++k) {
          const int c = lane + 32 * k;
          x[k] = c < n_elig ? xscale * row[c] : (c == c_i ? xd : -INFINITY);
        }
        const float tau = entmax_tau_warp<NV, KIND>(x, e);
#pragma unroll
        for (int k = 0; k < NV; ++k) wacc[k] += entmax_pow<KIND>(fmaxf(x[k] - tau, 0.f), e);
      }
      __syncthreads();
    }
  }
  const float invG = 1.f / (float)G;
  const size_t row = ((size_t)bg * seq + pos0 + warp);
  float* wr = w + row * n_c;
  const int nw = (n_c + 31) >> 5;
  uint32_t* mr = mask + row * nw;
  if (packed) {
    // compact form: the routed chunks of the row in increasing order
    int base = 0;
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int c = lane + 32 * k;
      const bool act = c < n_c && c < c_i && wacc[k] > 0.f;
      const unsigned bits = __ballot_sync(0xffffffffu, act);
      if (act) {
        const int at = base + __popc(bits & ((1u << lane) - 1u));
        wr[at] = wacc[k] * invG;
        if (index) index[row * n_c + at] = c;
      }
      if (k < nw && lane == 0) mr[k] = bits;
      base += __popc(bits);
    }
    if (count && lane == 0) count[row] = base;
    return;
  }
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int c = lane + 32 * k;
    // a row of the first chunk with the diagonal candidate: weight 1 on it
    if (c < n_c) wr[c] = diag && n_elig == 0 ? (c == c_i ? 1.f : 0.f) : wacc[k] * invG;
  }
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int c = lane + 32 * k;
    const unsigned bits = __ballot_sync(0xffffffffu, c < n_c && c < c_i && wacc[k] > 0.f);
    if (k < nw && lane == (k & 31)) mr[k] = bits;
  }
}

template <typename T, int D, int NV, int KIND>
cudaError_t launch_route_nv(const T* Q, const T* Kbar, float* w, uint32_t* mask, const T* K,
                            const float* qbar, int32_t* count, int32_t* index, int packed,
                            int batch, int n_q, int n_kv, int seq, int chunk, float xscale,
                            float e, cudaStream_t st) {
  const int n_c = (seq + chunk - 1) / chunk;
  const int LS = ((n_c + 7) & ~7) + 4;
  const size_t smem = (size_t)16 * LS * sizeof(float);
  auto kern = route_kernel<T, D, NV, KIND>;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const int n_bg = batch * n_kv;
  const unsigned grid = (unsigned)(n_bg * (seq / 8));
  kern<<<grid, 256, smem, st>>>(Q, Kbar, w, mask, K, qbar, count, index, packed, n_q, n_kv, seq,
                                chunk, n_c, seq / chunk, xscale, e, n_bg);
  return cudaGetLastError();
}

template <typename T, int D, int KIND>
cudaError_t launch_route_kind(const T* Q, const T* Kbar, float* w, uint32_t* mask, const T* K,
                              const float* qbar, int32_t* count, int32_t* index, int packed,
                              int batch, int n_q, int n_kv, int seq, int chunk, float xscale,
                              float e, cudaStream_t st) {
  const int n_c = (seq + chunk - 1) / chunk;
#define DASH_RNV(NV)                                                                            \
  launch_route_nv<T, D, NV, KIND>(Q, Kbar, w, mask, K, qbar, count, index, packed, batch, n_q,   \
                                  n_kv, seq, chunk, xscale, e, st)
  if (n_c <= 128) return DASH_RNV(4);
  if (n_c <= 256) return DASH_RNV(8);
  if (n_c <= 512) return DASH_RNV(16);
  if (n_c <= 1024) return DASH_RNV(32);
  return DASH_RNV(64);
#undef DASH_RNV
}

// K, qbar: non-null for estimate_diagonal (the keys and learned queries of
// stage 0), else both null.  packed: w is the compact form (count, index
// nullable), else dense.
template <typename T, int D>
cudaError_t launch_route(const T* Q, const T* Kbar, float* w, uint32_t* mask, const T* K,
                         const float* qbar, int batch, int n_q, int n_kv, int seq, int chunk,
                         float alpha, float gamma, cudaStream_t st, bool packed = false,
                         int32_t* count = nullptr, int32_t* index = nullptr) {
  const float xscale = (alpha - 1.f) * gamma;
  const float e = 1.f / (alpha - 1.f);
  const int pk = packed ? 1 : 0;
  if (alpha == 1.5f)
    return launch_route_kind<T, D, kEntmax15>(Q, Kbar, w, mask, K, qbar, count, index, pk, batch,
                                               n_q, n_kv, seq, chunk, xscale, e, st);
  if (alpha == 2.f)
    return launch_route_kind<T, D, kSparsemax>(Q, Kbar, w, mask, K, qbar, count, index, pk, batch,
                                                n_q, n_kv, seq, chunk, xscale, e, st);
  return launch_route_kind<T, D, kEntmaxGeneric>(Q, Kbar, w, mask, K, qbar, count, index, pk,
                                                  batch, n_q, n_kv, seq, chunk, xscale, e, st);
}

}  // namespace dash
