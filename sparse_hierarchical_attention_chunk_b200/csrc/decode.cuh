// Decode: one new query per sequence against a cached KV and summary cache.
//
// gist.science technical summary: "Fase 0" (a complete chunk's summary is
// fixed and cached, so decoding never recomputes it) and "Belangrijkste
// Bijdragen" item 4 (the kernels support incremental decoding); the
// decoding gain is reported in the memory-bound regime ("Efficiëntie").
// The new query sits at position L - 1 of an L-token cache; it routes over
// the summaries of chunks c < c_q = floor((L - 1) / B) and attends to the
// active chunks plus its own chunk (keys c_q B .. L - 1).  With a length per
// sequence (a batch of sequences at different points of their generation),
// L, c_q and the causal position are per sequence; the caches keep a common
// capacity.
//
// Three kernels on the caller's stream, each a programmatic dependent of the
// one before:
//
//   decode_route   one cluster of 8 CTAs per (b, h_kv).  CTA r computes the
//                  logits of all G <= 16 query heads for its slice of the
//                  chunks (mma.sync m16n8k16, the summary cache read once)
//                  and stores them, through distributed shared memory, in
//                  the CTA that owns the head (two heads per CTA).  Each head
//                  then finds its entmax threshold with four warps; the
//                  probabilities go back to the CTA owning each chunk, which
//                  forms the GQA mean w, the mask words and its part of the
//                  compact list of active chunks (with the log-prior bias);
//                  the list is stitched together by an exclusive scan of the
//                  8 slice counts, and the diagonal chunk is appended last.
//   decode_split   split-KV over the concatenation of all (b, h_kv) lists,
//                  cut into equal contiguous ranges (one per CTA) so that
//                  sequences with large supports do not serialise.  A
//                  producer warp streams the K/V blocks by TMA into a ring of
//                  stages; four warps run S and PV on mma.sync (M = 16 query
//                  heads).  A (b, h_kv) segment that lies inside one CTA is
//                  normalised and written by it; otherwise each CTA writes
//                  its (m, l, o) partial.  HBM-bound: every byte of the
//                  active K/V is read once.
//   decode_merge   o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s over the
//                  partials of each shared segment (one thread per row and
//                  4-float column).
#pragma once

#include <cooperative_groups.h>
#include <cuda.h>
#include "dash_common.cuh"
#include "route.cuh"
#include "tmap.cuh"

namespace dash {

constexpr int kDecodeMaxCtas = 512;
constexpr int kDecodeMaxItems = 288;       // K/V blocks staged per split CTA
constexpr int kRouteCluster = 8;           // CTAs per (b, h_kv) in decode_route
constexpr int kDecodeMaxChunks = 2048;

__host__ __device__ inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

struct DecodeWs {
  size_t off_list, off_bias, off_count, off_part, total;
};

__host__ __device__ inline DecodeWs decode_ws_layout(int batch, int n_kv, int L, int D, int chunk) {
  const int n_c = (L + chunk - 1) / chunk;
  const size_t n_bg = (size_t)batch * n_kv;
  DecodeWs w;
  size_t o = 0;
  w.off_list = o;  o = align256(o + n_bg * (n_c + 1) * sizeof(int));
  w.off_bias = o;  o = align256(o + n_bg * (n_c + 1) * sizeof(float));
  w.off_count = o; o = align256(o + n_bg * sizeof(int));
  w.off_part = o;  o = align256(o + (kDecodeMaxCtas + n_bg) * (size_t)16 * (D + 4) * sizeof(float));
  w.total = o;
  return w;
}

inline size_t decode_workspace_bytes(int batch, int n_q, int n_kv, int L, int D, int chunk) {
  (void)n_q;
  return decode_ws_layout(batch, n_kv, L, D, chunk).total;
}

// --------------------------------------------------------------------------
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3) : "r"(addr));
}

// byte offset of (row, 16-byte chunk cidx over the full head dim) in a
// TMA tile made of D/64 boxes of `rows` x 128 B with 128-byte swizzle
__device__ __forceinline__ uint32_t sw_off(int row, int cidx, int rows) {
  return (uint32_t)((cidx >> 3) * rows * 128 + row * 128 + (((cidx & 7) ^ (row & 7)) << 4));
}

// --------------------------------------------------------------------------
// reductions over a group of 4 warps (128 threads) with named barrier `id`;
// every thread adds the 4 warp totals in the same order, so all threads of
// the group hold bit-identical results and take the same branches
struct Group4 {
  float (*red)[4][4];                         // [2 parities][4 warps][4 values]
  int wg, lane, id, par;

  __device__ __forceinline__ void bar() const {
    asm volatile("bar.sync %0, 128;" ::"r"(id) : "memory");
  }
  __device__ __forceinline__ float4 sum4(float a, float b, float c, float d) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {        // four interleaved butterflies
      a += __shfl_xor_sync(0xffffffffu, a, o);
      b += __shfl_xor_sync(0xffffffffu, b, o);
      c += __shfl_xor_sync(0xffffffffu, c, o);
      d += __shfl_xor_sync(0xffffffffu, d, o);
    }
    if (lane == 0) *reinterpret_cast<float4*>(red[par][wg]) = make_float4(a, b, c, d);
    bar();
    float4 r = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const float4 v = *reinterpret_cast<const float4*>(red[par][i]);
      r.x += v.x;
      r.y += v.y;
      r.z += v.z;
      r.w += v.w;
    }
    par ^= 1;                                 // the next reduction writes the other half
    return r;
  }
  __device__ __forceinline__ float max1(float a) {
    a = warp_max(a);
    if (lane == 0) red[par][wg][0] = a;
    bar();
    float r = red[par][0][0];
#pragma unroll
    for (int i = 1; i < 4; ++i) r = fmaxf(r, red[par][i][0]);
    par ^= 1;
    return r;
  }
  __device__ __forceinline__ bool all(bool p) const {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred a, b;\n\t"
        "setp.ne.u32 a, %1, 0;\n\t"
        "bar.red.and.pred b, %2, 128, a;\n\t"
        "selp.u32 %0, 1, 0, b;\n\t}"
        : "=r"(r) : "r"((uint32_t)p), "r"(id) : "memory");
    return r != 0;
  }
};

// entmax threshold for the NV values held by each of the group's 128
// threads; the same iteration as the warp version in route.cuh (Newton on
// the e-norm from tau = max - 1, then the exact root on the support found
// for alpha = 1.5 / 2, kept only if self-consistent)
template <int NV, int KIND>
__device__ __forceinline__ float entmax_tau_group(const float (&x)[NV], float e, Group4& gr) {
  float m = -INFINITY;
#pragma unroll
  for (int k = 0; k < NV; ++k) m = fmaxf(m, x[k]);
  m = gr.max1(m);
  float tau = m - 1.f;
  for (int it = 0; it < 48; ++it) {
    float s0 = 0.f, s1 = 0.f;
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
    const float4 s = gr.sum4(s0, s1, 0.f, 0.f);
    const float f = s.x - 1.f;
    if (!(f > 0.f) || !(s.y > 0.f)) break;
    float step;
    if (KIND == kEntmax15) {
      step = (s.x - sqrtf(s.x)) / s.y;
    } else if (KIND == kSparsemax) {
      step = f / s.y;
    } else {
      const float nrm = ex2f(lg2f(s.x) / e);
      step = (nrm - 1.f) * s.x / (nrm * s.y);
    }
    const float nt = tau + step;
    if (!(nt > tau)) break;
    tau = nt;
    if (f < 1e-6f) break;
  }
  if (KIND == kEntmax15 || KIND == kSparsemax) {
    float d1 = 0.f, d2 = 0.f, kk = 0.f;
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const float d = x[k] - tau;
      if (d > 0.f) { d1 += d; d2 = fmaf(d, d, d2); kk += 1.f; }
    }
    const float4 s = gr.sum4(d1, d2, kk, 0.f);
    float tc = tau;
    bool cand = false;
    if (KIND == kEntmax15) {
      const float disc = s.x * s.x - s.z * (s.y - 1.f);
      if (s.z > 0.f && disc >= 0.f) { tc = tau + (s.y - 1.f) / (s.x + sqrtf(disc)); cand = true; }
    } else if (s.z > 0.f) {
      tc = tau + (s.x - 1.f) / s.z;
      cand = true;
    }
    if (cand) {                               // uniform: every thread holds the same sums
      bool ok = true;
#pragma unroll
      for (int k = 0; k < NV; ++k)
        if (x[k] > tau && !(x[k] > tc)) ok = false;
      if (gr.all(ok)) tau = tc;
    }
  }
  return tau;
}

struct DecodeRouteParams {
  const __nv_bfloat16* q;
  const __nv_bfloat16* Kbar;
  float* w;                    // nullable
  uint32_t* mask;              // nullable
  int* list;
  float* blist;
  int* counts;
  const int* lens;             // nullable: cache length per sequence (else L for all)
  // estimate_diagonal (diag != 0): the key cache (or page pool with
  // page_table) and the learned queries of stage 0
  const __nv_bfloat16* Kc;
  const float* qbar;
  const int* page_table;
  int max_pages, n_pages, diag;
  int n_q, n_kv, kbar_rows, n_c, L, chunk;
  float xscale, e, sigma;
};

template <int D, int KIND>
__global__ void __cluster_dims__(kRouteCluster, 1, 1) __launch_bounds__(256, 1)
decode_route_kernel(const __grid_constant__ CUtensorMap tmKb, const DecodeRouteParams prm) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  constexpr int NV = kDecodeMaxChunks / 128;  // values per thread in the entmax groups
  extern __shared__ uint8_t route_smem_raw[];
  // this CTA's slice of the summary cache (TMA, 128-byte swizzle; D / 64
  // boxes of CPC rows x 128 B)
  uint8_t* sKb = route_smem_raw + ((1024u - (smem_u32(route_smem_raw) & 1023u)) & 1023u);
  __shared__ __align__(8) uint64_t kb_bar[2];   // the two halves of the slice
  // logits of every head for this CTA's chunks (read by the heads' owners
  // after the first cluster barrier), then the staging of p of every head
  // for this CTA's chunks (pulled from the heads' owners)
  __shared__ __align__(16) float XP[16][256];
  __shared__ __align__(16) float Pl[2][kDecodeMaxChunks];   // p of the (<= 2) heads this CTA owns
  __shared__ float Xd[2];                     // estimate_diagonal: their diagonal logits
  __shared__ __align__(16) float red[2][2][4][4];   // float4 rows (Group4::sum4)
  __shared__ int cnt_all[kRouteCluster];
  __shared__ int wcnt[8];
  __shared__ float khat[D];                   // estimate_diagonal: the query chunk's summary

  const int r = (int)cluster.block_rank();
  const int bg = blockIdx.x / kRouteCluster;
  const int b = bg / prm.n_kv, g = bg % prm.n_kv;
  const int G = prm.n_q / prm.n_kv;
  const int HPC = (G + kRouteCluster - 1) / kRouteCluster;                  // heads per CTA
  const int CPC = (((prm.n_c + kRouteCluster - 1) / kRouteCluster) + 31) & ~31;  // chunks per CTA
  const int c0 = r * CPC;
  // this sequence's length; one outside [1, L] is recorded and clamped, so
  // that every access stays inside the caches
  int Lb = prm.L;
  if (prm.lens) {
    Lb = __ldg(prm.lens + b);
    if (Lb < 1 || Lb > prm.L) {
      if (r == 0 && threadIdx.x == 0) atomicOr(&g_dash_error, DASH_DEV_ERR_ARG);
      Lb = min(max(Lb, 1), prm.L);
    }
  }
  const int c_q = (Lb - 1) / prm.chunk;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // the split kernel that follows may start its launch now (it waits for
  // this grid's results before reading them)
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int rows_here = max(0, min(CPC, c_q - c0));   // eligible chunks of this slice
  if (tid == 0) {
    mbar_init(&kb_bar[0], 1);
    mbar_init(&kb_bar[1], 1);
    fence_mbar_init();
  }
  __syncthreads();
  if (tid == 0 && rows_here > 0) {
    tma_prefetch_desc(&tmKb);
    // two halves of CPC / 2 rows (a multiple of 16, so 1024-byte aligned in
    // the swizzled tile): the first half's logits start while the second
    // half is still in flight
    // (the second half only when it holds eligible chunks: the warp whose
    // first row of that half is eligible waits for it, so no copy is left
    // in flight when the CTA exits)
#pragma unroll
    for (int hf = 0; hf < (rows_here > CPC / 2 ? 2 : 1); ++hf) {
      mbar_arrive_expect_tx(&kb_bar[hf], (uint32_t)((D / 64) * (CPC / 2) * 128));
#pragma unroll
      for (int kb = 0; kb < D / 64; ++kb)
        tma_load_2d(sKb + kb * CPC * 128 + hf * (CPC / 2) * 128, &tmKb, &kb_bar[hf], kb * 64,
                    bg * prm.kbar_rows + c0 + hf * (CPC / 2));
    }
  }

  // ---- logits of all heads for chunks [c0, c0 + CPC), kept in this CTA
  {
    constexpr int KS = D / 16;
    const int gi = lane >> 2, t = lane & 3;
    const bool v0 = gi < G, v1 = gi + 8 < G;
    const uint32_t* q0 = reinterpret_cast<const uint32_t*>(
        prm.q + ((size_t)b * prm.n_q + g * G + (v0 ? gi : 0)) * D);
    const uint32_t* q1 = reinterpret_cast<const uint32_t*>(
        prm.q + ((size_t)b * prm.n_q + g * G + (v1 ? gi + 8 : 0)) * D);
    uint32_t qa[KS][4];
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      qa[kk][0] = v0 ? __ldg(q0 + kk * 8 + t) : 0u;
      qa[kk][1] = v1 ? __ldg(q1 + kk * 8 + t) : 0u;
      qa[kk][2] = v0 ? __ldg(q0 + kk * 8 + t + 4) : 0u;
      qa[kk][3] = v1 ? __ldg(q1 + kk * 8 + t + 4) : 0u;
    }
    // warp-uniform: the ldmatrix / mma below need the whole warp
    const bool have = __all_sync(0xffffffffu, rows_here > 0 && mbar_wait(&kb_bar[0], 0, nullptr));
    if (have) {
      const uint32_t sb = smem_u32(sKb);
      bool second = false;                        // waited for the second half
      // pairs of n-tiles (16 chunks) per warp step; B fragments by ldmatrix
      for (int pr = warp; pr * 16 < rows_here; pr += 8) {
        if (pr * 16 >= CPC / 2 && !second) {
          if (!__all_sync(0xffffffffu, mbar_wait(&kb_bar[1], 0, nullptr))) break;
          second = true;
        }
        float acc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        const int mi = lane >> 3, rr = lane & 7;
        const int row = pr * 16 + ((mi >> 1) << 3) + rr;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(sb + sw_off(row, 2 * kk + (mi & 1), CPC), b0, b1, b2, b3);
          mma_bf16_16816(acc[0], qa[kk], b0, b1);
          mma_bf16_16816(acc[1], qa[kk], b2, b3);
        }
        // chunks past c_q keep whatever the MMA gave: the owners read only
        // the eligible ones
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          const int cl = pr * 16 + hf * 8 + 2 * t;
          if (v0) *reinterpret_cast<float2*>(&XP[gi][cl]) =
              make_float2(acc[hf][0] * prm.xscale, acc[hf][1] * prm.xscale);
          if (v1) *reinterpret_cast<float2*>(&XP[gi + 8][cl]) =
              make_float2(acc[hf][2] * prm.xscale, acc[hf][3] * prm.xscale);
        }
      }
    }
  }
  // ---- estimate_diagonal: the query's own chunk c_q as one more candidate,
  // its logit against stage 0's summary of the cache rows c_q B .. L_b - 1,
  // computed by the CTA that owns each head (Xd[slot])
  const bool dg = prm.diag != 0 && c_q > 0;
  if (dg && r * HPC < G) {                      // uniform over the CTA
    if (warp == 0) {
      const __nv_bfloat16* rows;
      if (prm.page_table) {
        int pg = __ldg(prm.page_table + (size_t)b * prm.max_pages + c_q);
        if (pg < 0 || pg >= prm.n_pages) {
          if (lane == 0) atomicOr(&g_dash_error, DASH_DEV_ERR_ARG);
          pg = 0;
        }
        rows = prm.Kc + ((size_t)pg * prm.n_kv + g) * prm.chunk * D;
      } else {
        rows = prm.Kc + ((size_t)bg * prm.L + (size_t)c_q * prm.chunk) * D;
      }
      summarize_chunk_warp<__nv_bfloat16, D, 4, float>(rows, prm.qbar + g * D, khat,
                                                      Lb - c_q * prm.chunk, lane);
    }
    __syncthreads();
    const int h = r * HPC + warp;
    if (warp < HPC && h < G) {
      const __nv_bfloat16* qh = prm.q + ((size_t)b * prm.n_q + g * G + h) * D;
      float acc = 0.f;
      for (int j = lane; j < D; j += 32) acc = fmaf(__bfloat162float(qh[j]), khat[j], acc);
      acc = warp_sum(acc);
      if (lane == 0) Xd[warp] = acc * prm.xscale;
    }
  }
  cluster.sync();

  // ---- entmax of the owned heads, four warps per head.  Each thread pulls
  // its 16 logits as four float4 (chunks 512 k + 4 tg .. + 3; a CTA's slice
  // is a multiple of 32 chunks, so a float4 never straddles two CTAs) and
  // keeps p in this CTA (Pl) for the chunk owners to pull.
  const int n_cand = c_q + (dg ? 1 : 0);        // candidates: eligible chunks (+ the diagonal)
  {
    const int slot = warp >> 2;
    const int h = r * HPC + slot;
    if (slot < HPC && h < G && c_q > 0) {       // uniform over the 4-warp group
      const int tg = tid & 127;
      float x[NV];
#pragma unroll
      for (int k = 0; k < NV / 4; ++k) {
        const int c = 512 * k + 4 * tg;
        float4 v = make_float4(-INFINITY, -INFINITY, -INFINITY, -INFINITY);
        if (c < c_q) {
          const int owner = c / CPC;
          v = *cluster.map_shared_rank(reinterpret_cast<float4*>(&XP[h][c - owner * CPC]), owner);
        }
        x[4 * k + 0] = c + 0 < c_q ? v.x : (dg && c + 0 == c_q ? Xd[slot] : -INFINITY);
        x[4 * k + 1] = c + 1 < c_q ? v.y : (dg && c + 1 == c_q ? Xd[slot] : -INFINITY);
        x[4 * k + 2] = c + 2 < c_q ? v.z : (dg && c + 2 == c_q ? Xd[slot] : -INFINITY);
        x[4 * k + 3] = c + 3 < c_q ? v.w : (dg && c + 3 == c_q ? Xd[slot] : -INFINITY);
      }
      Group4 gr{red[slot], warp & 3, lane, 1 + slot, 0};
      const float tau = entmax_tau_group<NV, KIND>(x, prm.e, gr);
#pragma unroll
      for (int k = 0; k < NV / 4; ++k) {
        const int c = 512 * k + 4 * tg;
        if (c < n_cand) {
          float4 pv;
          pv.x = entmax_pow<KIND>(fmaxf(x[4 * k + 0] - tau, 0.f), prm.e);
          pv.y = entmax_pow<KIND>(fmaxf(x[4 * k + 1] - tau, 0.f), prm.e);
          pv.z = entmax_pow<KIND>(fmaxf(x[4 * k + 2] - tau, 0.f), prm.e);
          pv.w = entmax_pow<KIND>(fmaxf(x[4 * k + 3] - tau, 0.f), prm.e);
          *reinterpret_cast<float4*>(&Pl[slot][c]) = pv;
        }
      }
    }
  }
  cluster.sync();

  // ---- p of every head for this CTA's chunks, pulled from the heads' owners
  // (float4, in the order of the heads) into XP, whose logits are no longer
  // read by anyone after the barrier above
  {
    // at most 16 heads x 64 float4 = 4 per thread: all four loads are in
    // flight before any is stored
    const int lim = min(CPC, n_cand - c0);      // this slice's candidate chunks
    const int q4 = (lim + 3) >> 2;
    float4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = tid + u * 256;
      if (i < G * q4) {
        const int hh = i / q4, cl = 4 * (i % q4);
        v[u] = *cluster.map_shared_rank(reinterpret_cast<const float4*>(&Pl[hh % HPC][c0 + cl]), hh / HPC);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = tid + u * 256;
      if (i < G * q4) *reinterpret_cast<float4*>(&XP[i / q4][4 * (i % q4)]) = v[u];
    }
  }
  __syncthreads();

  // ---- GQA mean, mask words and this CTA's part of the active list
  const int c = c0 + tid;
  float wv = 0.f;
  bool act = false;
  if (tid < CPC && c < prm.n_c) {
    if (c < n_cand) {
      float s = 0.f;
      for (int hh = 0; hh < G; ++hh) s += XP[hh][tid];
      wv = s / (float)G;
    } else if (prm.diag && c == c_q && c_q == 0) {
      wv = 1.f;                                   // the diagonal is the only candidate
    }
    if (prm.w) prm.w[(size_t)bg * prm.n_c + c] = wv;
    act = wv > 0.f && c < c_q;                    // the query's own chunk is never routed
  }
  const unsigned bal = __ballot_sync(0xffffffffu, act);
  const int nw = (prm.n_c + 31) >> 5;
  if (lane == 0 && prm.mask && tid < CPC && c < prm.n_c) prm.mask[(size_t)bg * nw + (c >> 5)] = bal;
  if (lane == 0) wcnt[warp] = __popc(bal);
  __syncthreads();
  if (tid == 0) {
    int tot = 0;
    for (int i = 0; i < 8; ++i) tot += wcnt[i];
    for (int rr = 0; rr < kRouteCluster; ++rr) *cluster.map_shared_rank(&cnt_all[r], rr) = tot;
  }
  cluster.sync();
  int off = 0;
  for (int rr = 0; rr < r; ++rr) off += cnt_all[rr];
  int woff = 0;
  for (int i = 0; i < warp; ++i) woff += wcnt[i];
  int* lst = prm.list + (size_t)bg * (prm.n_c + 1);
  float* bl = prm.blist + (size_t)bg * (prm.n_c + 1);
  if (act) {
    const int at = off + woff + __popc(bal & ((1u << lane) - 1u));
    lst[at] = c;
    bl[at] = prm.sigma == 0.f ? 0.f : prm.sigma * lg2f(wv);   // log2 units, as the scores
  }
  if (r == kRouteCluster - 1 && tid == 0) {
    const int total = off + cnt_all[r];
    lst[total] = c_q;                            // the query's own chunk, causal, bias 0
    bl[total] = 0.f;
    prm.counts[bg] = total + 1;
  }
}

// named barrier over the 128 consumer threads (warps 0-3)
__device__ __forceinline__ void consumers_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ bool consumers_all(bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\t"
      "setp.ne.u32 a, %1, 0;\n\t"
      "bar.red.and.pred b, 1, 128, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r) : "r"((uint32_t)p) : "memory");
  return r != 0;
}

struct DecodeSplitParams {
  const __nv_bfloat16* q;
  const int* list;
  const float* blist;
  const int* counts;
  float* part;
  __nv_bfloat16* o;
  float* lse;                  // nullable
  const int* lens;             // nullable: cache length per sequence (else L for all)
  const int* page_table;       // nullable: [batch][max_pages] pool page of each chunk
  int max_pages, n_pages;
  int n_q, n_kv, n_bg, L, n_c, chunk;
  float scale_log2;
};

// largest k in [0, NC) whose range [k T / NC, (k + 1) T / NC) starts at or before x
__device__ __forceinline__ long long split_cta_of(long long x, long long T, long long NC) {
  long long k = (x * NC) / T;
  while (k + 1 < NC && ((k + 1) * T) / NC <= x) ++k;
  return k;
}

template <int BLK, int D>
struct SplitCfg {
  static constexpr int KV_BOX = BLK * 128;
  static constexpr int KV_BYTES = KV_BOX * (D / 64);
  static constexpr int STAGE = 2 * KV_BYTES;                      // K then V
  static constexpr int RED_BYTES = 4 * 16 * (D + 4) * 4;
  static constexpr int NS_FIT = (200 * 1024 - RED_BYTES) / STAGE;
  static constexpr int NS = NS_FIT > 8 ? 8 : (NS_FIT < 2 ? 2 : NS_FIT);
  static constexpr size_t SMEM = (size_t)NS * STAGE + RED_BYTES + 1024;
};

template <int BLK, int D>
__global__ void __launch_bounds__(160, 1) decode_split_kernel(
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const DecodeSplitParams prm) {
  using C = SplitCfg<BLK, D>;
  constexpr int NS = C::NS;
  constexpr int KV_BOX = C::KV_BOX, KV_BYTES = C::KV_BYTES, STAGE = C::STAGE;
  constexpr int KPW = BLK / 4;                      // keys per consumer warp
  constexpr int NT = KPW / 8;                       // S n-tiles per warp
  constexpr int KS = D / 16;
  constexpr int DT = D / 8;                         // O n-tiles
  constexpr int RS = D + 4;                         // partial row: o[D], m, l, 2 pad (16-B rows)
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned by pointer arithmetic on the shared array, so that the
  // compiler keeps the shared address space (and emits shared loads)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  float* red = reinterpret_cast<float*>(smem + NS * STAGE);     // [4 warps][16 rows][RS]
  __shared__ float fac[16][4], rowM[16], rowL[16];
  __shared__ __align__(8) uint64_t full[NS], empty[NS];
  __shared__ int seg_start[65];
  __shared__ int seg_cq[64], seg_pos[64];        // query chunk and position of each (b, h_kv)
  __shared__ int it_c[kDecodeMaxItems];
  __shared__ float it_b[kDecodeMaxItems];
  __shared__ uint8_t it_g[kDecodeMaxItems];
  __shared__ int it_r[kDecodeMaxItems];              // first K/V row of the block in the tensor maps
  __shared__ int s_T, s_issued, s_consumed;
  __shared__ volatile int abort_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gi = lane >> 2, t = lane & 3;
  const int G = prm.n_q / prm.n_kv;
  const int n_bg = prm.n_bg;
  if (tid == 0) {
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  // launched early behind the routing kernel: its lists are read below
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // decode_merge may be scheduled now; it waits for this whole grid
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");

  // segment starts: exclusive prefix of the per-(b, h_kv) list lengths (n_bg <= 64)
  if (warp == 0) {
    int base = 0;
    for (int i0 = 0; i0 < n_bg; i0 += 32) {
      const int i = i0 + lane;
      const int v = i < n_bg ? prm.counts[i] : 0;
      int incl = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += u;
      }
      if (i < n_bg) seg_start[i] = base + incl - v;
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      seg_start[n_bg] = base;
      s_T = base;
    }
  } else if (warp == 1) {
    for (int i = lane; i < n_bg; i += 32) {
      // lengths were checked (and recorded if bad) by decode_route
      const int Lb = prm.lens ? min(max(__ldg(prm.lens + i / prm.n_kv), 1), prm.L) : prm.L;
      seg_cq[i] = (Lb - 1) / prm.chunk;
      seg_pos[i] = Lb - 1;
    }
  }
  if (tid == 32) {
    abort_s = 0;
    s_issued = 0;
    s_consumed = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 4);
    }
    fence_mbar_init();
  }
  __syncthreads();
  const long long T = s_T;
  const long long NC = min((long long)gridDim.x, T);
  const long long k = blockIdx.x;
  if (k >= NC) return;                               // whole CTA, before any further barrier
  const long long s0 = k * T / NC, s1 = (k + 1) * T / NC;
  const int n_items = (int)(s1 - s0);
  if (n_items > kDecodeMaxItems) {                   // the host sizes the grid so this cannot happen
    if (tid == 0) atomicOr(&g_dash_error, DASH_DEV_ERR_LIMIT);
    return;
  }
  // stage this CTA's items: chunk, bias and (b, h_kv) of each K/V block
  for (int i = tid; i < n_items; i += blockDim.x) {
    const long long x = s0 + i;
    int lo = 0, hi = n_bg - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (seg_start[mid] <= x) lo = mid;
      else hi = mid - 1;
    }
    const int li = (int)(x - seg_start[lo]);
    const int cc = prm.list[(size_t)lo * (prm.n_c + 1) + li];
    it_c[i] = cc;
    it_b[i] = prm.blist[(size_t)lo * (prm.n_c + 1) + li];
    it_g[i] = (uint8_t)lo;
    if (prm.page_table) {
      // paged caches: chunk cc of this sequence lives in pool page pg, whose
      // rows for KV head h start at (pg H_kv + h) B; a page id outside the
      // pool is recorded and replaced by page 0 (every access stays inside)
      int pg = __ldg(prm.page_table + (size_t)(lo / prm.n_kv) * prm.max_pages + cc);
      if (pg < 0 || pg >= prm.n_pages) {
        atomicOr(&g_dash_error, DASH_DEV_ERR_ARG);
        pg = 0;
      }
      it_r[i] = (pg * prm.n_kv + lo % prm.n_kv) * BLK;
    } else {
      it_r[i] = lo * prm.L + cc * BLK;
    }
  }
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      // every K/V block is read once per step: keep it from evicting the
      // partials and list the merge reads back (measured: ~8 us less per
      // step on 8 x 128k caches)
      const uint64_t pol = l2_evict_first_policy();
      int it = 0;
      for (; it < n_items; ++it) {
        const int s = it % NS;
        if (it >= NS && !mbar_wait(&empty[s], ((it / NS) - 1) & 1, &abort_s)) break;
        const int row = it_r[it];
        uint8_t* st = smem + s * STAGE;
        mbar_arrive_expect_tx(&full[s], STAGE);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          tma_load_2d_hint(st + kb * KV_BOX, &tmK, &full[s], kb * 64, row, pol);
          tma_load_2d_hint(st + KV_BYTES + kb * KV_BOX, &tmV, &full[s], kb * 64, row, pol);
        }
      }
      s_issued = it;
    }
  } else {
    // ------------------------------------------------------------ consumers
    uint32_t qa[KS][4];
    float oacc[DT][4];
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    int cur = -1;

    auto load_q = [&](int bgi) {
      const int b = bgi / prm.n_kv, g = bgi % prm.n_kv;
      const bool v0 = gi < G, v1 = gi + 8 < G;
      const uint32_t* q0 = reinterpret_cast<const uint32_t*>(prm.q + ((size_t)b * prm.n_q + g * G + (v0 ? gi : 0)) * D);
      const uint32_t* q1 = reinterpret_cast<const uint32_t*>(prm.q + ((size_t)b * prm.n_q + g * G + (v1 ? gi + 8 : 0)) * D);
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        qa[kk][0] = v0 ? __ldg(q0 + kk * 8 + t) : 0u;
        qa[kk][1] = v1 ? __ldg(q1 + kk * 8 + t) : 0u;
        qa[kk][2] = v0 ? __ldg(q0 + kk * 8 + t + 4) : 0u;
        qa[kk][3] = v1 ? __ldg(q1 + kk * 8 + t + 4) : 0u;
      }
#pragma unroll
      for (int dt = 0; dt < DT; ++dt) oacc[dt][0] = oacc[dt][1] = oacc[dt][2] = oacc[dt][3] = 0.f;
      m0 = m1 = -INFINITY;
      l0 = l1 = 0.f;
    };

    // merge the 4 warps' (m, l, o) of segment bgi; write the output if the
    // segment is all here, else this CTA's partial (decode_merge combines them)
    auto flush = [&](int bgi) {
      // this warp's (m, l, o) -> red
      float* rw = red + warp * 16 * RS;
      const float lt0 = l0 + __shfl_xor_sync(0xffffffffu, l0, 1);
      const float lr0 = lt0 + __shfl_xor_sync(0xffffffffu, lt0, 2);
      const float lt1 = l1 + __shfl_xor_sync(0xffffffffu, l1, 1);
      const float lr1 = lt1 + __shfl_xor_sync(0xffffffffu, lt1, 2);
#pragma unroll
      for (int dt = 0; dt < DT; ++dt) {
        *reinterpret_cast<float2*>(rw + gi * RS + dt * 8 + 2 * t) = make_float2(oacc[dt][0], oacc[dt][1]);
        *reinterpret_cast<float2*>(rw + (gi + 8) * RS + dt * 8 + 2 * t) = make_float2(oacc[dt][2], oacc[dt][3]);
      }
      if (t == 0) {
        rw[gi * RS + D] = m0;
        rw[gi * RS + D + 1] = lr0;
        rw[(gi + 8) * RS + D] = m1;
        rw[(gi + 8) * RS + D + 1] = lr1;
      }
      consumers_sync();
      // per row: the merged max and the 4 warps' factors
      if (tid < 64) {
        const int r = tid >> 2, w2 = tid & 3;
        const float mw = red[(w2 * 16 + r) * RS + D];
        float M = fmaxf(mw, __shfl_xor_sync(0xffffffffu, mw, 1));
        M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, 2));
        const float f = M == -INFINITY ? 0.f : ex2f(mw - M);
        float lw = f * red[(w2 * 16 + r) * RS + D + 1];
        lw += __shfl_xor_sync(0xffffffffu, lw, 1);
        lw += __shfl_xor_sync(0xffffffffu, lw, 2);
        fac[r][w2] = f;
        if (w2 == 0) {
          rowM[r] = M;
          rowL[r] = lw;
        }
      }
      consumers_sync();
      const int seg0 = seg_start[bgi], seg1 = seg_start[bgi + 1];
      const bool whole = seg0 >= s0 && seg1 <= s1;
      const int b = bgi / prm.n_kv, g = bgi % prm.n_kv;
      float* slot = prm.part + (size_t)(k + bgi) * 16 * RS;
      for (int i = tid; i < G * (D / 4); i += 128) {
        const int r = i / (D / 4), c = (i % (D / 4)) * 4;
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int w2 = 0; w2 < 4; ++w2) {
          const float f = fac[r][w2];
          const float4 v = *reinterpret_cast<const float4*>(red + (w2 * 16 + r) * RS + c);
          o.x = fmaf(f, v.x, o.x);
          o.y = fmaf(f, v.y, o.y);
          o.z = fmaf(f, v.z, o.z);
          o.w = fmaf(f, v.w, o.w);
        }
        if (whole) {
          const size_t orow = (size_t)b * prm.n_q + g * G + r;
          const float inv = 1.f / rowL[r];
          uint2 pk;
          pk.x = pack_bf16x2(o.x * inv, o.y * inv);
          pk.y = pack_bf16x2(o.z * inv, o.w * inv);
          *reinterpret_cast<uint2*>(prm.o + orow * D + c) = pk;
          if (c == 0 && prm.lse) prm.lse[orow] = (rowM[r] + log2f(rowL[r])) * 0.69314718055994531f;
        } else {
          *reinterpret_cast<float4*>(slot + r * RS + c) = o;
          if (c == 0) {
            slot[r * RS + D] = rowM[r];
            slot[r * RS + D + 1] = rowL[r];
          }
        }
      }
      consumers_sync();                          // red may be reused
    };

    const float scale = prm.scale_log2;
    bool ok = true;
    int it = 0;
    for (; it < n_items; ++it) {
      const int s = it % NS;
      ok = consumers_all(mbar_wait(&full[s], (it / NS) & 1, &abort_s));
      if (!ok) break;                            // uniform over the consumers
      const int bgi = it_g[it];
      if (bgi != cur) {
        if (cur >= 0) flush(cur);
        load_q(bgi);
        cur = bgi;
      }
      const int c = it_c[it];
      const float bias = it_b[it];
      const bool diag = c == seg_cq[bgi];
      const int pos = seg_pos[bgi];
      const uint32_t sK = smem_u32(smem + s * STAGE);
      const uint32_t sV = sK + KV_BYTES;
      const int key0 = warp * KPW;
      // S = q K^T for this warp's KPW keys
      // (even and odd k-steps in separate accumulators: shorter MMA chains)
      float sacc[NT][4], sodd[NT][4];
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) sacc[nt][i] = sodd[nt][i] = 0.f;
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
#pragma unroll
        for (int np = 0; np < NT / 2; ++np) {
          const int mi = lane >> 3, rr = lane & 7;
          const int key = key0 + np * 16 + ((mi >> 1) << 3) + rr;
          const int cidx = 2 * kk + (mi & 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4(sK + sw_off(key, cidx, BLK), b0, b1, b2, b3);
          mma_bf16_16816((kk & 1) ? sodd[2 * np] : sacc[2 * np], qa[kk], b0, b1);
          mma_bf16_16816((kk & 1) ? sodd[2 * np + 1] : sacc[2 * np + 1], qa[kk], b2, b3);
        }
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int i = 0; i < 4; ++i) sacc[nt][i] += sodd[nt][i];
      // bias / causal mask, online softmax (rows gi and gi + 8)
      float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
          const int kpos = c * BLK + key0 + nt * 8 + 2 * t + e2;
          const bool okk = !diag || kpos <= pos;
          sacc[nt][e2] = okk ? fmaf(sacc[nt][e2], scale, bias) : -INFINITY;
          sacc[nt][2 + e2] = okk ? fmaf(sacc[nt][2 + e2], scale, bias) : -INFINITY;
          mx0 = fmaxf(mx0, sacc[nt][e2]);
          mx1 = fmaxf(mx1, sacc[nt][2 + e2]);
        }
      }
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
      mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
      mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
      const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
      const float mu0 = mn0 == -INFINITY ? 0.f : mn0, mu1 = mn1 == -INFINITY ? 0.f : mn1;
      const float cr0 = ex2f(m0 - mu0), cr1 = ex2f(m1 - mu1);
      m0 = mn0;
      m1 = mn1;
      l0 *= cr0;
      l1 *= cr1;
#pragma unroll
      for (int dt = 0; dt < DT; ++dt) {
        oacc[dt][0] *= cr0;
        oacc[dt][1] *= cr0;
        oacc[dt][2] *= cr1;
        oacc[dt][3] *= cr1;
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) {
        sacc[nt][0] = ex2f(sacc[nt][0] - mu0);
        sacc[nt][1] = ex2f(sacc[nt][1] - mu0);
        sacc[nt][2] = ex2f(sacc[nt][2] - mu1);
        sacc[nt][3] = ex2f(sacc[nt][3] - mu1);
        l0 += sacc[nt][0] + sacc[nt][1];
        l1 += sacc[nt][2] + sacc[nt][3];
      }
      // O += P V for this warp's keys (16 keys per k-step)
#pragma unroll
      for (int ks = 0; ks < KPW / 16; ++ks) {
        uint32_t pa[4];
        pa[0] = pack_bf16x2(sacc[2 * ks][0], sacc[2 * ks][1]);
        pa[1] = pack_bf16x2(sacc[2 * ks][2], sacc[2 * ks][3]);
        pa[2] = pack_bf16x2(sacc[2 * ks + 1][0], sacc[2 * ks + 1][1]);
        pa[3] = pack_bf16x2(sacc[2 * ks + 1][2], sacc[2 * ks + 1][3]);
        const int mi = lane >> 3, rr = lane & 7;
        const int key = key0 + ks * 16 + ((mi & 1) << 3) + rr;
#pragma unroll
        for (int dp = 0; dp < DT / 2; ++dp) {
          const int cidx = 2 * dp + (mi >> 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(sV + sw_off(key, cidx, BLK), b0, b1, b2, b3);
          mma_bf16_16816(oacc[2 * dp], pa, b0, b1);
          mma_bf16_16816(oacc[2 * dp + 1], pa, b2, b3);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);     // this warp is done with stage s
    }
    if (ok && cur >= 0) flush(cur);
    if (tid == 0) s_consumed = it;
  }
  __syncthreads();
  if (tid == 128 && abort_s) {
    // let copies still in flight land before the CTA exits
    for (int i = s_consumed; i < s_issued; ++i) mbar_wait(&full[i % NS], (i / NS) & 1, nullptr);
  }
}

// --------------------------------------------------------------------------
// Merge of the split-KV partials: o = sum_s 2^(m_s - M) o_s / sum_s 2^(m_s - M) l_s
// over the CTAs that shared one (b, h_kv), M the row max (scores in log2 units).
struct DecodeMergeParams {
  const int* counts;
  const float* part;
  __nv_bfloat16* o;
  float* lse;                  // nullable
  int n_q, n_kv, n_bg, n_split;
};

// grid: n_bg x (16 / rows per CTA); thread (row, float4 column); a segment that
// one split CTA held whole was written by it and is skipped here
template <int D>
__global__ void __launch_bounds__(128) decode_merge_kernel(const DecodeMergeParams prm) {
  constexpr int TPR = D / 4;                        // threads per row
  constexpr int RPC = 128 / TPR;                    // rows per CTA
  constexpr int RS = D + 4;
  constexpr int SLOT = 16 * RS;
  constexpr int U = 8;                              // partials in flight per thread
  const int nrg = 16 / RPC;
  const int bgi = blockIdx.x / nrg;
  const int r = (blockIdx.x % nrg) * RPC + threadIdx.x / TPR;
  const int c4 = threadIdx.x % TPR, lane = threadIdx.x & 31;
  const int G = prm.n_q / prm.n_kv;
  asm volatile("griddepcontrol.wait;" ::: "memory");   // the split grid is complete
  // start of segment bgi, start of the next, and the total: each warp scans the counts
  int seg0 = 0, seg1 = 0, T = 0;
  for (int i0 = 0; i0 < prm.n_bg; i0 += 32) {
    const int i = i0 + lane;
    const int v = i < prm.n_bg ? __ldcg(prm.counts + i) : 0;
    int incl = v;
#pragma unroll
    for (int o2 = 1; o2 < 32; o2 <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o2);
      if (lane >= o2) incl += u;
    }
    const int excl = T + incl - v;
    if (bgi >= i0 && bgi < i0 + 32) {
      seg0 = __shfl_sync(0xffffffffu, excl, bgi - i0);
      seg1 = seg0 + __shfl_sync(0xffffffffu, v, bgi - i0);
    }
    T += __shfl_sync(0xffffffffu, incl, 31);
  }
  const long long NC = min((long long)prm.n_split, (long long)T);
  const long long kf = split_cta_of(seg0, T, NC), kl = split_cta_of(seg1 - 1, T, NC);
  if (kf == kl || r >= G) return;
  const int n = (int)(kl - kf + 1);
  const float* base = prm.part + (size_t)(kf + bgi) * SLOT + (size_t)r * RS;
  float M = -INFINITY, Ls = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int p0 = 0; p0 < n; p0 += U) {
    float mk[U], lk[U];
    float4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float* q = base + (size_t)min(p0 + u, n - 1) * SLOT;   // in bounds; weight 0 past n
      mk[u] = p0 + u < n ? __ldcg(q + D) : -INFINITY;
      lk[u] = __ldcg(q + D + 1);
      v[u] = __ldcg(reinterpret_cast<const float4*>(q) + c4);
    }
    float mb = M;
#pragma unroll
    for (int u = 0; u < U; ++u) mb = fmaxf(mb, mk[u]);
    const float sc = M == -INFINITY ? 0.f : ex2f(M - mb);
    acc.x *= sc;
    acc.y *= sc;
    acc.z *= sc;
    acc.w *= sc;
    Ls *= sc;
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float f = mk[u] == -INFINITY ? 0.f : ex2f(mk[u] - mb);
      acc.x = fmaf(f, v[u].x, acc.x);
      acc.y = fmaf(f, v[u].y, acc.y);
      acc.z = fmaf(f, v[u].z, acc.z);
      acc.w = fmaf(f, v[u].w, acc.w);
      Ls = fmaf(f, lk[u], Ls);
    }
    M = mb;
  }
  const int b = bgi / prm.n_kv, g = bgi % prm.n_kv;
  const size_t orow = (size_t)b * prm.n_q + g * G + r;
  const float inv = 1.f / Ls;
  uint2 pk;
  pk.x = pack_bf16x2(acc.x * inv, acc.y * inv);
  pk.y = pack_bf16x2(acc.z * inv, acc.w * inv);
  *reinterpret_cast<uint2*>(prm.o + orow * D + 4 * c4) = pk;
  if (c4 == 0 && prm.lse) prm.lse[orow] = (M + log2f(Ls)) * 0.69314718055994531f;
}

// --------------------------------------------------------------------------
inline int route_cpc(int n_c) {                  // chunks per CTA of decode_route
  return (((n_c + kRouteCluster - 1) / kRouteCluster) + 31) & ~31;
}

template <int D, int KIND>
cudaError_t launch_decode_route_k(const CUtensorMap& tkb, const DecodeRouteParams& prm, int n_bg,
                                  cudaStream_t st) {
  auto kern = decode_route_kernel<D, KIND>;
  const size_t smem = (size_t)(D / 64) * route_cpc(prm.n_c) * 128 + 1024;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  kern<<<(unsigned)(n_bg * kRouteCluster), 256, smem, st>>>(tkb, prm);
  return cudaGetLastError();
}

template <int D>
cudaError_t launch_decode_route(const CUtensorMap& tkb, const DecodeRouteParams& prm, int n_bg,
                                float alpha, cudaStream_t st) {
  if (alpha == 1.5f) return launch_decode_route_k<D, kEntmax15>(tkb, prm, n_bg, st);
  if (alpha == 2.f) return launch_decode_route_k<D, kSparsemax>(tkb, prm, n_bg, st);
  return launch_decode_route_k<D, kEntmaxGeneric>(tkb, prm, n_bg, st);
}

template <int BLK, int D>
cudaError_t launch_decode_split(const CUtensorMap& tk, const CUtensorMap& tv,
                                const DecodeSplitParams& prm, int n_ctas, cudaStream_t st) {
  auto kern = decode_split_kernel<BLK, D>;
  const size_t smem = SplitCfg<BLK, D>::SMEM;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  // programmatic dependent launch: the CTAs may be scheduled while the
  // routing kernel finishes; they wait for it (griddepcontrol.wait) before
  // reading its output
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)n_ctas);
  cfg.blockDim = dim3(160);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, tk, tv, prm);
}

template <int D>
cudaError_t launch_decode_merge(const DecodeMergeParams& prm, cudaStream_t st) {
  // programmatic dependent of the split grid, like that one of the routing grid
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(prm.n_bg * (16 / (128 / (D / 4)))));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, decode_merge_kernel<D>, prm);
}

// number of split CTAs: one per SM, more if a CTA would otherwise get more
// than kDecodeMaxItems blocks in the densest case (every chunk active)
inline int decode_split_ctas(int n_bg, int c_q, int sms) {
  const long long t_max = (long long)n_bg * (c_q + 1);
  const long long need = (t_max + kDecodeMaxItems - 2) / (kDecodeMaxItems - 1);
  long long n = sms > need ? sms : need;
  return (int)(n < kDecodeMaxCtas ? n : kDecodeMaxCtas);
}

// lens: nullable device array [batch] of cache lengths (1 <= lens[b] <= L);
// L is then the caches' capacity.  page_table: nullable device array
// [batch][max_pages]; with it Kc and Vc are page pools [n_pages][n_kv][chunk][D]
// and chunk c of sequence b is pool page page_table[b][c].
// qbar: nullable; non-null turns on estimate_diagonal (the learned queries of
// stage 0, [n_kv][D] fp32).
inline int run_decode(int batch, int n_q, int n_kv, int L, int D, int chunk, float alpha,
                      float gamma, float sigma, const int* lens, const int* page_table,
                      int max_pages, int n_pages, const __nv_bfloat16* q, const __nv_bfloat16* Kc,
                      const __nv_bfloat16* Vc, const __nv_bfloat16* Kbar, const float* qbar,
                      __nv_bfloat16* o, float* lse, float* w, uint32_t* mask, void* workspace,
                      cudaStream_t st) {
  const int n_bg = batch * n_kv;
  const int n_c = (L + chunk - 1) / chunk;
  if (n_bg > 64 || n_c > kDecodeMaxChunks || n_q / n_kv > 16) return 2;   // DASH_ERR_UNSUPPORTED
  const int c_q = (L - 1) / chunk;
  const DecodeWs lay = decode_ws_layout(batch, n_kv, L, D, chunk);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* list = reinterpret_cast<int*>(ws + lay.off_list);
  float* blist = reinterpret_cast<float*>(ws + lay.off_bias);
  int* counts = reinterpret_cast<int*>(ws + lay.off_count);
  float* part = reinterpret_cast<float*>(ws + lay.off_part);

  DecodeRouteParams rp;
  rp.q = q;
  rp.Kbar = Kbar;
  rp.w = w;
  rp.mask = mask;
  rp.list = list;
  rp.blist = blist;
  rp.counts = counts;
  rp.n_q = n_q;
  rp.n_kv = n_kv;
  rp.lens = lens;
  rp.Kc = Kc;
  rp.qbar = qbar;
  rp.page_table = page_table;
  rp.max_pages = max_pages;
  rp.n_pages = n_pages;
  rp.diag = qbar != nullptr;
  rp.kbar_rows = L / chunk;
  rp.n_c = n_c;
  rp.L = L;
  rp.chunk = chunk;
  rp.xscale = (alpha - 1.f) * gamma;
  rp.e = 1.f / (alpha - 1.f);
  rp.sigma = sigma;
  CUtensorMap tkb;
  {
    // rows of every (b, h_kv); with no complete chunk at all the map is
    // never read, and is laid over the K cache so that it stays valid
    const uint64_t rows = (uint64_t)n_bg * (L / chunk);
    const uint64_t dims[2] = {(uint64_t)D, rows > 0 ? rows : 1};
    const uint64_t str[1] = {(uint64_t)D * 2};
    const uint32_t box[2] = {64, (uint32_t)route_cpc(n_c) / 2};   // half a slice
    if (!make_tmap(&tkb, rows > 0 ? Kbar : Kc, 2, dims, str, box)) return 3;
  }
  cudaError_t e = D == 128 ? launch_decode_route<128>(tkb, rp, n_bg, alpha, st)
                           : launch_decode_route<64>(tkb, rp, n_bg, alpha, st);
  if (e != cudaSuccess) return 3;

  CUtensorMap tk, tv;
  const uint64_t kv_rows = page_table ? (uint64_t)n_pages * n_kv * chunk : (uint64_t)n_bg * L;
  const uint64_t dims[2] = {(uint64_t)D, kv_rows};
  const uint64_t str[1] = {(uint64_t)D * 2};
  const uint32_t box[2] = {64, (uint32_t)chunk};
  if (!make_tmap(&tk, Kc, 2, dims, str, box) || !make_tmap(&tv, Vc, 2, dims, str, box)) return 3;
  // SM count of the current device, read on every call (a host-side lookup):
  // the split grid is sized for the device the call runs on
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || sms < 1)
    return 3;
  const int n_ctas = decode_split_ctas(n_bg, c_q, sms);
  DecodeSplitParams prm;
  prm.q = q;
  prm.list = list;
  prm.blist = blist;
  prm.counts = counts;
  prm.part = part;
  prm.o = o;
  prm.lse = lse;
  prm.n_q = n_q;
  prm.n_kv = n_kv;
  prm.n_bg = n_bg;
  prm.lens = lens;
  prm.page_table = page_table;
  prm.max_pages = max_pages;
  prm.n_pages = n_pages;
  prm.L = L;
  prm.n_c = n_c;
  prm.chunk = chunk;
  prm.scale_log2 = 1.4426950408889634f / sqrtf((float)D);
  if (chunk == 64)
    e = D == 128 ? launch_decode_split<64, 128>(tk, tv, prm, n_ctas, st) : launch_decode_split<64, 64>(tk, tv, prm, n_ctas, st);
  else
    e = D == 128 ? launch_decode_split<128, 128>(tk, tv, prm, n_ctas, st) : launch_decode_split<128, 64>(tk, tv, prm, n_ctas, st);
  if (e != cudaSuccess) return 3;
  DecodeMergeParams mp;
  mp.counts = counts;
  mp.part = part;
  mp.o = o;
  mp.lse = lse;
  mp.n_q = n_q;
  mp.n_kv = n_kv;
  mp.n_bg = n_bg;
  mp.n_split = n_ctas;
  e = D == 128 ? launch_decode_merge<128>(mp, st) : launch_decode_merge<64>(mp, st);
  return e == cudaSuccess ? 0 : 3;
}

}  // namespace dash
