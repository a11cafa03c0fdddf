// Stage 2 backward on tcgen05 (bf16, G query heads per KV head, d = 128).
//
// The chain rule of the prior-induced block-sparse softmax of the
// gist.science technical summary, "Fase 2" (the pages state end-to-end
// differentiability, "Belangrijkste Bijdragen" item 1, and print no
// gradients).  For a row (position i, query head h) and its active keys j,
// s_j = q.k_j / sqrt(d) + beta_j, p = softmax(s) (recomputed from the
// forward's log-normaliser), with the cotangent do and D = do.o:
//   dp_j = do.v_j,  ds_j = p_j (dp_j - D),
//   dq = sum_j ds_j k_j / sqrt(d),  dk_j = sum_rows ds_j q / sqrt(d),
//   dv_j = sum_rows p_j do,  dw_c = sigma / w_c sum_{j in c, group heads} ds_j.
// Two kernels, neither with atomics on dQ, dK or dV (every output element is
// written by one CTA, in a fixed order):
//
//   attn_bwd_dq_kernel   query-major, like the forward: one tile of M = 128
//       rows (P = 128 / G positions x G heads) per CTA walks the diagonal
//       chunk and the union of its positions' routed chunks in 64-key blocks.
//       Per block: S = Q K^T and dP = dO V^T (TS-MMAs, Q and dO copied into
//       TMEM), then eight row warps (two per TMEM lane quarter, 32 keys each)
//       form P and dS (written as bf16 over S) and the row sums of dS (-> dw,
//       summed over the heads of a position by shuffles; the two halves'
//       shares added to the zeroed dw), then dQ += dS K (K as the MN-major
//       operand).  S/dP are double-buffered, so block n+1's S and dP run
//       while block n's dS is formed.  Also writes D = dO . O per row and each
//       tile's routed union, for the key-major kernel.
//   attn_bwd_dkv_kernel  key-major: one CTA per 128 keys (one 128-key chunk
//       or a pair of 64-key chunks; with few key blocks, a share of the
//       block's tiles) walks the query tiles whose rows attend to those keys
//       (the tiles of the keys' own chunks, causal, and every later tile whose
//       routed union holds them).  Per tile: S^T = K Q^T and dP^T = V dO^T
//       (SS-MMAs, M = 128 keys, N = 128 rows), P^T and dS^T by eight key
//       warps (a row table of exponent offsets and D in shared memory), then
//       dV += P^T dO and dK += dS^T Q with the accumulators in TMEM for the
//       whole walk; the next tile's S^T and dP^T are interleaved with them.
#pragma once

#include <cuda.h>
#include <type_traits>
#include "dash_common.cuh"
#include "tmem_wide.cuh"
#include "attn_tc.cuh"

namespace dash {

struct BwdParams {
  const float* w;
  const uint32_t* mask;
  const float* lse;
  const __nv_bfloat16* O;
  const __nv_bfloat16* dO;
  float* dQ;
  float* dK;
  float* dV;
  float* dw;             // nullable
  float* Drow;           // [b, n_q, seq]: dO . O (written by the dQ kernel)
  uint32_t* tmask;       // [b * n_kv, nw, n_tiles]: each tile's routed union (dQ kernel)
  float* part;           // [n_split, b * n_kv * seq, 256]: partial dK | dV (n_split > 1)
  int n_q, n_kv, seq, chunk, n_c, nw, G, lgG, P, n_tiles, n_bg, n_split;
  float sigma, scale_log2, scale;
};

// ---------------------------------------------------------------------------
// dQ and dw
// ---------------------------------------------------------------------------
// K / V ring depth of the dQ kernel: block n + 2's S and dP are issued right
// after block n's dQ, so its slot must have been freed two steps earlier
constexpr int kBwdDqStages = 4;

// Eight row warps: two per TMEM lane quarter, each taking 32 of a block's 64
// keys; then the producer and the MMA issuer.
constexpr int kBwdRowWarps = 8;

// Two 32-column TMEM loads (32 lanes x 32-bit) and one wait, in one asm
// statement so that no use of the registers is scheduled before the data.
__device__ __forceinline__ void tmem_ld32x2(uint32_t ta, uint32_t tb, float (&va)[32], float (&vb)[32]) {
  uint32_t r[64];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%64];\n\t"
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%65];\n\t"
      "tcgen05.wait::ld.sync.aligned;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]),
        "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]),
        "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]),
        "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]),
        "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(ta), "r"(tb)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    va[i] = __uint_as_float(r[i]);
    vb[i] = __uint_as_float(r[32 + i]);
  }
}

template <int CHUNK>
__global__ void __launch_bounds__(32 * (kBwdRowWarps + 2), 1) attn_bwd_dq_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const BwdParams prm) {
  constexpr int D = 128;
  constexpr int BLK = 64;                        // keys per block
  constexpr int SB = CHUNK / BLK;                // sub-blocks per chunk
  constexpr int NS = kBwdDqStages;               // K / V ring depth
  constexpr int QBOX = 128 * 128;                // 128 rows x 128 B
  constexpr int T_BYTES = 2 * QBOX;              // one 128 x 128 bf16 tile
  constexpr int KV_BOX = BLK * 128;
  constexpr int KV_BYTES = 2 * KV_BOX;
  // TMEM columns: Q | dO (bf16 pairs) | dQ (fp32) | S, dP of buffer 0 | of buffer 1
  constexpr uint32_t TM_Q = 0, TM_DO = 64, TM_DQ = 128, TM_BUF = 256;
  constexpr int NRT = 32 * kBwdRowWarps;         // row threads
  constexpr int W_PROD = kBwdRowWarps, W_MMA = kBwdRowWarps + 1;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned by pointer arithmetic on the shared array, so that the
  // compiler keeps the shared address space (and emits shared loads)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sdO = sQ + T_BYTES;
  uint8_t* sK = sdO + T_BYTES;
  uint8_t* sV = sK + NS * KV_BYTES;
  int* list = reinterpret_cast<int*>(sV + NS * KV_BYTES);                // [n_c + 1]
  uint32_t* mrows = reinterpret_cast<uint32_t*>(list + prm.n_c + 1);     // [P][nw]
  float* w_sm = reinterpret_cast<float*>(mrows + prm.P * prm.nw);        // [NS][P]

  __shared__ __align__(8) uint64_t bar_qd, bar_qd_tm, bar_s_full[2], bar_ds_full[2], bar_fin;
  __shared__ float dpart[2][128];                // the halves of each row's dO . O
  __shared__ __align__(8) uint64_t bar_k_full[NS], bar_k_empty[NS], bar_v_full[NS], bar_v_empty[NS];
  __shared__ uint32_t tmem_slot;
  __shared__ int nb_s;
  __shared__ volatile int abort_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = prm.n_tiles - 1 - (int)(blockIdx.x % prm.n_tiles);   // late tiles first
  const int bg = (int)(blockIdx.x / prm.n_tiles);
  const int b = bg / prm.n_kv, g = bg % prm.n_kv;
  const int P = prm.P, G = prm.G;
  const int pos0 = tile * P;
  const int c_i = pos0 / CHUNK;
  const int n_wl = min(P, 32);

  if (warp == W_MMA) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_qd, 1);
    mbar_init(&bar_qd_tm, NRT);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar_s_full[t], 1);
      mbar_init(&bar_ds_full[t], NRT);
    }
    mbar_init(&bar_fin, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_k_full[s], 1);
      mbar_init(&bar_k_empty[s], 1);
      mbar_init(&bar_v_full[s], 1 + n_wl);
      mbar_init(&bar_v_empty[s], 1);
    }
    abort_s = 0;
    fence_mbar_init();
  }
  const size_t row0 = (size_t)bg * prm.seq + pos0;
  for (int i = tid; i < P * prm.nw; i += blockDim.x) mrows[i] = prm.mask[row0 * prm.nw + i];
  __syncthreads();
  // block list: the diagonal chunk, then the union of the routed chunks c < c_i
  if (warp == 0) {
    int base = 1;
    for (int k0 = 0; k0 < prm.nw; k0 += 32) {
      const int k = k0 + lane;
      uint32_t u = 0;
      if (k < prm.nw && k * 32 < c_i) {
        for (int p = 0; p < P; ++p) u |= mrows[p * prm.nw + k];
        const int rem = c_i - k * 32;
        if (rem < 32) u &= (1u << rem) - 1u;
      }
      if (k < prm.nw) prm.tmask[((size_t)bg * prm.nw + k) * prm.n_tiles + tile] = u;
      const int cnt = __popc(u);
      int incl = cnt;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      int at = base + incl - cnt;
      while (u) {
        const int bit = __ffs(u) - 1;
        u &= u - 1;
        list[at++] = k * 32 + bit;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) {
      list[0] = c_i;
      nb_s = base;
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const int nb = nb_s;
  // walk: the diagonal chunk's sub-blocks (the second only if a position
  // reaches it), then SB sub-blocks per routed chunk
  const int diag_lo = c_i * CHUNK;
  const int n_diag = (SB == 2 && pos0 + P - 1 >= diag_lo + BLK) ? 2 : 1;
  const int nbb = n_diag + (nb - 1) * SB;
  struct Entry { int j, c, sb; };
  auto entry = [&](int jj) {
    Entry e;
    if (jj < n_diag) {
      e.j = 0; e.c = c_i; e.sb = jj;
    } else {
      const int r = jj - n_diag;
      e.j = 1 + r / SB; e.sb = r % SB; e.c = list[e.j];
    }
    return e;
  };

  if (warp == W_PROD) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar_qd, 2 * T_BYTES);
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) {
        tma_load_3d(sQ + kb * QBOX, &tmQ, &bar_qd, kb * 64, b * prm.n_q + g * G, pos0);
        tma_load_3d(sdO + kb * QBOX, &tmdO, &bar_qd, kb * 64, b * prm.n_q + g * G, pos0);
      }
    }
    int issued_k = 0, issued_v = 0;
    for (int j = 0; j < nbb; ++j) {
      const int s = j % NS;
      const uint32_t par = ((j / NS) & 1) ^ 1;
      const Entry en = entry(j);
      const int krow = bg * prm.seq + en.c * CHUNK + en.sb * BLK;
      int okw = lane == 0 ? (int)mbar_wait(&bar_k_empty[s], par, &abort_s) : 0;
      if (!__shfl_sync(0xffffffffu, okw, 0)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar_k_full[s], KV_BYTES);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
          tma_load_2d(sK + s * KV_BYTES + kb * KV_BOX, &tmK, &bar_k_full[s], kb * 64, krow);
      }
      issued_k = j + 1;
      okw = lane == 0 ? (int)mbar_wait(&bar_v_empty[s], par, &abort_s) : 0;
      if (!__shfl_sync(0xffffffffu, okw, 0)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar_v_full[s], KV_BYTES);
#pragma unroll
        for (int kb = 0; kb < 2; ++kb)
          tma_load_2d(sV + s * KV_BYTES + kb * KV_BOX, &tmV, &bar_v_full[s], kb * 64, krow);
      }
      if (lane < n_wl) {
        for (int q = lane; q < P; q += 32)
          cp_async_4(w_sm + s * P + q, prm.w + (row0 + q) * prm.n_c + en.c);
        cp_async_arrive_noinc(&bar_v_full[s]);
      }
      issued_v = j + 1;
    }
    if (abort_s) {
      if (lane == 0) {
        for (int j = (issued_k > NS ? issued_k - NS : 0); j < issued_k; ++j)
          mbar_wait(&bar_k_full[j % NS], (j / NS) & 1, nullptr);
        for (int j = (issued_v > NS ? issued_v - NS : 0); j < issued_v; ++j)
          mbar_wait(&bar_v_full[j % NS], (j / NS) & 1, nullptr);
      }
      cp_async_wait_all();
    }
  } else if (warp == W_MMA) {
    // ------------------------------------------------------------ MMA issuer
    // S(n), dP(n) into buffer n & 1; after block n's dS: dQ(n), then S(n+2),
    // dP(n+2) into the same buffer (in issue order, after dQ(n) read dS(n)).
    constexpr uint32_t idS = idesc_bf16_f32(128, BLK, 0, 0);
    constexpr uint32_t idQ = idesc_bf16_f32(128, D, 0, 1);
    const bool leader = elect_one();
    const uint64_t dK0 = sw128_desc(smem_u32(sK), 16, 1024);
    const uint64_t dV0 = sw128_desc(smem_u32(sV), 16, 1024);
    const uint64_t dKmn0 = sw128_desc(smem_u32(sK), KV_BOX, 1024);   // K as the MN-major operand
    int n_s = 0, n_q = 0;
    auto wait_all = [&](uint64_t* bar, uint32_t par) {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, &abort_s));
    };
    auto issue_sdp = [&](int n) {            // S(n), dP(n); K(n), V(n) loaded
      const int s = n % NS;
      const uint32_t buf = tmem + TM_BUF + (uint32_t)(n & 1) * 128;
      const uint64_t dk = dK0 + (uint64_t)((s * KV_BYTES) >> 4);
      const uint64_t dv = dV0 + (uint64_t)((s * KV_BYTES) >> 4);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offk = (kk >> 2) * KV_BOX + (kk & 3) * 32;
          tc_mma_ts(buf, tmem + TM_Q + kk * 8, dk + (offk >> 4), idS, kk > 0 ? 1u : 0u);
        }
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offk = (kk >> 2) * KV_BOX + (kk & 3) * 32;
          tc_mma_ts(buf + 64, tmem + TM_DO + kk * 8, dv + (offk >> 4), idS, kk > 0 ? 1u : 0u);
        }
        tc_commit(&bar_s_full[n & 1]);
      }
      __syncwarp();
      ++n_s;
    };
    bool ok = wait_all(&bar_qd_tm, 0);
    for (int n = 0; ok && n < 2 && n < nbb; ++n) {
      if (!(ok = wait_all(&bar_k_full[n % NS], (n / NS) & 1) &&
                 wait_all(&bar_v_full[n % NS], (n / NS) & 1)))
        break;
      tc_fence_after();
      issue_sdp(n);
    }
    for (int n = 0; ok && n < nbb; ++n) {
      const int s = n % NS;
      if (!(ok = wait_all(&bar_ds_full[n & 1], (n >> 1) & 1))) break;
      tc_fence_after();
      const uint32_t ds = tmem + TM_BUF + (uint32_t)(n & 1) * 128;   // dS(n), bf16 pairs
      const uint64_t dkm = dKmn0 + (uint64_t)((s * KV_BYTES) >> 4);
      if (leader) {
        // dS of keys 32 h + 16 j .. (packed) sits at columns 32 h + 8 j
#pragma unroll
        for (int kk = 0; kk < BLK / 16; ++kk)
          tc_mma_ts(tmem + TM_DQ, ds + (kk >> 1) * 32 + (kk & 1) * 8, dkm + (uint64_t)((kk * 2048) >> 4), idQ,
                    (n > 0 || kk > 0) ? 1u : 0u);
        tc_commit(&bar_k_empty[s]);
        tc_commit(&bar_v_empty[s]);
        if (n + 1 == nbb) tc_commit(&bar_fin);
      }
      __syncwarp();
      ++n_q;
      if (n + 2 < nbb) {
        const int s2 = (n + 2) % NS;
        if (!(ok = wait_all(&bar_k_full[s2], ((n + 2) / NS) & 1) &&
                   wait_all(&bar_v_full[s2], ((n + 2) / NS) & 1)))
          break;
        tc_fence_after();
        issue_sdp(n + 2);
      }
    }
    if (abort_s && lane == 0) {
      if (n_s > 0) mbar_wait(&bar_s_full[(n_s - 1) & 1], ((n_s - 1) >> 1) & 1, nullptr);
      if (n_q > 0) mbar_wait(&bar_k_empty[(n_q - 1) % NS], ((n_q - 1) / NS) & 1, nullptr);
    }
  } else {
    // ------------------------------------------------------------ rows (warps 0-7)
    const int r = tid & 127;                   // row = TMEM lane
    const int half = warp >> 2;                // keys 32 half .. 32 half + 31 of each block
    const int p = r / G, hq = r % G;
    const int pos = pos0 + p;
    const int qh = g * G + hq;
    const uint32_t tlane = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t* mrow = mrows + p * prm.nw;
    const size_t qrow = ((size_t)b * prm.n_q + qh) * prm.seq + pos;
    const float sigma = prm.sigma;
    const float lse2 = prm.lse[qrow] * 1.4426950408889634f;
    const uint64_t sc2 = f2_pack(prm.scale_log2, prm.scale_log2);
    // D = dO . O of this row (fp32; each half takes 64 of the d columns), also
    // kept for the key-major kernel
    {
      // all sixteen 16-byte loads in flight at once: one round trip
      const uint4* orow = reinterpret_cast<const uint4*>(prm.O + qrow * D + half * 64);
      const uint4* drow = reinterpret_cast<const uint4*>(prm.dO + qrow * D + half * 64);
      uint4 a[8], c[8];
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        a[v] = __ldg(orow + v);
        c[v] = __ldg(drow + v);
      }
      float dpp = 0.f;
#pragma unroll
      for (int v = 0; v < 8; ++v) {
        const __nv_bfloat16* xa = reinterpret_cast<const __nv_bfloat16*>(&a[v]);
        const __nv_bfloat16* xc = reinterpret_cast<const __nv_bfloat16*>(&c[v]);
#pragma unroll
        for (int e = 0; e < 8; ++e) dpp = fmaf(__bfloat162float(xa[e]), __bfloat162float(xc[e]), dpp);
      }
      dpart[half][r] = dpp;
    }
    asm volatile("bar.sync 1, %0;" ::"r"(NRT) : "memory");
    const float Dr = dpart[0][r] + dpart[1][r];
    if (half == 0) prm.Drow[qrow] = Dr;
    // waits are made warp-uniform: the TMEM loads / stores and shuffles below
    // are warp-collective
    bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_qd, 0, &abort_s));
    // Q (half 0) and dO (half 1) rows: shared memory (TMA, 128-byte swizzle)
    // -> TMEM as bf16 pairs
    if (ok) {
      const uint8_t* base = (half ? sdO : sQ) + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
      for (int kb = 0; kb < 2; ++kb) {
        uint32_t h0[16], h1[16];
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) {
          const uint4 q4 = *reinterpret_cast<const uint4*>(base + kb * QBOX + ((ch ^ (r & 7)) << 4));
          uint32_t* dst = ch < 4 ? h0 + ch * 4 : h1 + (ch - 4) * 4;
          dst[0] = q4.x;
          dst[1] = q4.y;
          dst[2] = q4.z;
          dst[3] = q4.w;
        }
        const uint32_t dst = tmem + tlane + (half ? TM_DO : TM_Q) + kb * 32;
        tmem_st16u(dst, h0);
        tmem_st16u(dst + 16, h1);
      }
      tmem_wait_st();
    }
    tc_fence_before();
    mbar_arrive(&bar_qd_tm);
    float dsum_chunk = 0.f;                    // this half's dS summed over a routed chunk
    for (int n = 0; ok && n < nbb; ++n) {
      const Entry en = entry(n);
      const int c = en.c;
      const bool act = en.j == 0 || ((mrow[c >> 5] >> (c & 31)) & 1u);
      if (!__all_sync(0xffffffffu, mbar_wait(&bar_s_full[n & 1], (n >> 1) & 1, &abort_s))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float bias = 0.f;
      float wc = 0.f;
      if (en.j > 0) {
        // the routing weights of block n (cp.async, counted on V's barrier)
        if (!__all_sync(0xffffffffu, mbar_wait(&bar_v_full[n % NS], (n / NS) & 1, &abort_s))) {
          ok = false;
          break;
        }
        if (!act) {
          bias = -INFINITY;
        } else {
          wc = w_sm[(n % NS) * P + p];
          if (sigma != 0.f) bias = sigma * lg2f(wc);
        }
      }
      const uint32_t tb = tmem + tlane + TM_BUF + (uint32_t)(n & 1) * 128 + half * 32;
      float dsum = 0.f;
      if (!__any_sync(0xffffffffu, act)) {
        uint32_t z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0u;
        tmem_st16u(tb, z);
      } else {
        float sv[32], dp[32];
        tmem_ld32x2(tb, tb + 64, sv, dp);
        // causal on the diagonal: key k of the block is seen iff k <= lim
        const int lim = (en.j == 0 ? pos - (c * CHUNK + en.sb * BLK) : BLK) - half * 32;
        const uint64_t off2 = f2_pack(bias - lse2, bias - lse2);
        const uint64_t D2 = f2_pack(Dr, Dr);
        // p = 2^(s * scale + off): 3 of every 8 pairs on the FMA pipe
        // (exp2_poly2), the rest on the special-function unit
        constexpr uint32_t kPolyPairs = 0x52u;   // pairs 1, 4, 6 of each 8
        uint32_t pk[16];
        // the causal test only on the diagonal chunk's blocks
        auto pass = [&](auto causal) {
#pragma unroll
          for (int k2 = 0; k2 < 16; ++k2) {
            const uint64_t x = f2_fma(f2_pack(sv[2 * k2], sv[2 * k2 + 1]), sc2, off2);
            float e0, e1;
            if ((kPolyPairs >> (k2 & 7)) & 1u) {
              exp2_poly2(x, e0, e1);
            } else {
              float x0, x1;
              f2_unpack(x, x0, x1);
              e0 = ex2f(x0);
              e1 = ex2f(x1);
            }
            if (decltype(causal)::value) {
              e0 = 2 * k2 <= lim ? e0 : 0.f;
              e1 = 2 * k2 + 1 <= lim ? e1 : 0.f;
            }
            const uint64_t d2 = f2_mul(f2_pack(e0, e1), f2_sub(f2_pack(dp[2 * k2], dp[2 * k2 + 1]), D2));
            float a0, a1;
            f2_unpack(d2, a0, a1);
            dsum += a0 + a1;
            pk[k2] = pack_bf16x2(a0, a1);
          }
        };
        if (lim < 31) pass(std::true_type{});
        else pass(std::false_type{});
        tmem_st16u(tb, pk);                    // dS over the half's own S columns
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_ds_full[n & 1]);
      // dw of a routed chunk: sigma / w times the sum of dS over its keys and
      // the heads of the position (adjacent lanes); the two halves' shares
      // are added to the zeroed dw (two terms: the sum does not depend on
      // their order)
      if (en.j > 0 && prm.dw && sigma != 0.f) {
        dsum_chunk += dsum;
        if (en.sb == SB - 1) {
          float tot = dsum_chunk;
          for (int o = 1; o < G; o <<= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
          if (hq == 0 && act && wc > 0.f)
            atomicAdd(prm.dw + ((size_t)bg * prm.seq + pos) * prm.n_c + c, sigma / wc * tot);
          dsum_chunk = 0.f;
        }
      }
    }
    // dQ: half 0 writes columns 0-63, half 1 columns 64-127
    if (ok && __all_sync(0xffffffffu, mbar_wait(&bar_fin, 0, &abort_s))) {
      tc_fence_after();
      float* drow = prm.dQ + qrow * D + half * 64;
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        float o[32];
        tmem_ld32(tmem + tlane + TM_DQ + half * 64 + cc * 32, o);
        float4* dst = reinterpret_cast<float4*>(drow + cc * 32);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          dst[q4] = make_float4(o[4 * q4] * prm.scale, o[4 * q4 + 1] * prm.scale,
                                o[4 * q4 + 2] * prm.scale, o[4 * q4 + 3] * prm.scale);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

inline size_t attn_bwd_dq_smem_bytes(int n_c, int nw, int P) {
  return (size_t)2 * 2 * 128 * 128 + (size_t)kBwdDqStages * 2 * 2 * 64 * 128 + (size_t)(n_c + 1) * 4 +
         (size_t)P * nw * 4 + (size_t)kBwdDqStages * P * 4 + 1024 + 64;
}

// ---------------------------------------------------------------------------
// dK and dV
// ---------------------------------------------------------------------------

// Named barrier `id` over `count` threads that also ANDs a predicate across them.
__device__ __forceinline__ bool bar_and(int id, int count, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.and.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r) : "r"((uint32_t)v), "r"(id), "r"(count) : "memory");
  return r != 0;
}

// Per 128-key CTA and 128-row query tile, in the tensor core's order:
//   S^T(n) = K Q^T, dP^T(n) = V dO^T   (SS-MMAs, N = 128)
//   dV += P^T(n) dO                      once the key threads wrote P^T over S^T
//   S^T(n + 1)                           over P^T, behind dV(n)
//   dK += dS^T(n) Q                      once they wrote dS^T over dP^T
//   dP^T(n + 1)                          over dS^T, behind dK(n)
// so the key threads form P^T(n + 1) while the tensor core runs dK(n) and
// dP^T(n + 1), and dS^T(n) while it runs dV(n) and S^T(n + 1).  Eight key
// warps: two per TMEM lane quarter, each taking 64 of the tile's 128 rows;
// each keeps its P in registers between the two passes.
// Q and dO tiles share one ring of four 32 KB slots.  A tile frees its dO
// after dV and its Q after dK, half a tile later; the tile two ahead takes
// the first freed slot for its Q and the second for its dO, so each load
// has about a whole tile of lead: tile m's Q sits in slot 2 (m & 1) +
// ((m >> 1) & 1), its dO in the other slot of that pair.
constexpr int kBwdDkvSlots = 4;
__device__ __forceinline__ int bwd_qslot(int m) { return 2 * (m & 1) + ((m >> 1) & 1); }
__device__ __forceinline__ int bwd_dslot(int m) { return 2 * (m & 1) + 1 - ((m >> 1) & 1); }
constexpr int kBwdKeyWarps = 8;
// A key block's tile list is split over n_split CTAs (interleaved by tile
// ordinal) when there are few key blocks: about four waves of 148 SMs.
constexpr int kBwdSplitTarget = 4 * 148;
constexpr int kBwdMaxSplit = 8;

inline int attn_bwd_n_split(int n_kb, int n_bg) {
  const int units = n_kb * n_bg;
  int s = (kBwdSplitTarget + units - 1) / units;
  return s < 1 ? 1 : (s > kBwdMaxSplit ? kBwdMaxSplit : s);
}

// Row data of a query tile staged beside its Q and dO (lse and D
// head-major, as they lie in memory; each position's routing weights of the
// key block's chunks and the mask word holding them), and the row table the
// key threads build from it: per chunk of the block and row t = p G + h of
// the tile, the exponent offset (log2 units: routing bias minus lse; -inf
// where the row does not see the chunk) and D.
template <int NCK>
struct BwdTile {
  float lse[128];
  float D[128];
  float w[32][2];
  uint32_t mword[32];
  float off[NCK][128];
  float dd[NCK][128];
};

template <int CHUNK>
__global__ void __launch_bounds__(32 * (kBwdKeyWarps + 2), 1) attn_bwd_dkv_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmdO,
    const __grid_constant__ CUtensorMap tmK, const __grid_constant__ CUtensorMap tmV,
    const BwdParams prm) {
  constexpr int D = 128;
  constexpr int KB = 128;                        // keys per CTA
  constexpr int NCK = KB / CHUNK;                // chunks per key block (2 or 1)
  constexpr int NSL = kBwdDkvSlots;
  constexpr int NKT = 32 * kBwdKeyWarps;         // key threads
  constexpr int W_PROD = kBwdKeyWarps, W_MMA = kBwdKeyWarps + 1;
  constexpr int QBOX = 128 * 128;                // 128 rows x 128 B
  constexpr int T_BYTES = 2 * QBOX;              // one 128 x 128 bf16 tile
  // TMEM columns: dK, dV accumulators | S^T (then P^T) | dP^T (then dS^T)
  constexpr uint32_t TM_DK = 0, TM_DV = 128, TM_S = 256, TM_DP = 384;
  using Tile = BwdTile<NCK>;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned by pointer arithmetic on the shared array, so that the
  // compiler keeps the shared address space (and emits shared loads)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sK = smem;                            // the block's keys (two 64-column boxes)
  uint8_t* sV = sK + T_BYTES;
  uint8_t* sT = sV + T_BYTES;                    // [NSL] Q / dO tile slots
  Tile* tiles = reinterpret_cast<Tile*>(sT + NSL * T_BYTES);   // [NSL] row data of a Q slot

  // per slot: filled (TMA bytes plus 32 producer-lane arrivals: the row
  // data's copies for a Q, plain arrivals for a dO) and freed (by the MMA)
  __shared__ __align__(8) uint64_t bar_kv, bar_full[NSL], bar_empty[NSL];
  __shared__ __align__(8) uint64_t bar_s_full, bar_dp_full, bar_p_full, bar_ds_full, bar_fin;
  __shared__ int slot_tile[NSL];                 // the tile whose Q a slot holds
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_kb = (prm.seq + KB - 1) / KB;      // the grid's key blocks (the last may be half)
  const int split = (int)(blockIdx.x % prm.n_split);
  const int kb = (int)((blockIdx.x / prm.n_split) % n_kb);   // early key blocks (the most tiles) first
  const int bg = (int)(blockIdx.x / prm.n_split / n_kb);
  const int b = bg / prm.n_kv, g = bg % prm.n_kv;
  const int P = prm.P, G = prm.G;
  const int kc0 = kb * NCK;                      // first chunk of the key block
  const int key0 = kb * KB;

  if (warp == W_MMA) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_kv, 1);
    for (int s = 0; s < NSL; ++s) {
      mbar_init(&bar_full[s], 1 + 32);
      mbar_init(&bar_empty[s], 1);
    }
    mbar_init(&bar_s_full, 1);
    mbar_init(&bar_dp_full, 1);
    mbar_init(&bar_p_full, NKT);
    mbar_init(&bar_ds_full, NKT);
    mbar_init(&bar_fin, 1);
    abort_s = 0;
    fence_mbar_init();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == W_PROD) {
    // ------------------------------------------------------------ producer
    // K, V of the key block once; then, in position order, every query tile
    // whose rows attend to a key of the block -- the tiles of the block's own
    // chunks (causal) and the later tiles whose routed union (written by the
    // dQ kernel) holds one of the block's chunks -- keeping the ordinals that
    // fall to this split.  A tile id of -1 ends the walk.
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar_kv, 2 * T_BYTES);
#pragma unroll
      for (int kb2 = 0; kb2 < 2; ++kb2) {
        tma_load_2d(sK + kb2 * QBOX, &tmK, &bar_kv, kb2 * 64, bg * prm.seq + key0);
        tma_load_2d(sV + kb2 * QBOX, &tmV, &bar_kv, kb2 * 64, bg * prm.seq + key0);
      }
    }
    const int tile0 = key0 / P;                  // first tile of the block's chunks
    const int tile_own = (key0 + KB) / P;        // first tile after them
    const int wsel = kc0 >> 5;                   // mask word holding the block's chunks
    uint32_t bsel = 0;
#pragma unroll
    for (int ck = 0; ck < NCK; ++ck) bsel |= 1u << ((kc0 + ck) & 31);
    const uint32_t* tm_row = prm.tmask + ((size_t)bg * prm.nw + wsel) * prm.n_tiles;
    int n_it = 0;                                // tiles whose Q was issued
    int n_do = 0;                                // tiles whose dO was issued
    int ord = 0;                                 // relevant tiles seen
    bool go = true;
    // slot x's fill for tile m: free once its previous use (tile m - 2) is done
    auto take = [&](int x, int m) {
      int okw = 1;
      if (m >= 2 && lane == 0) okw = (int)mbar_wait(&bar_empty[x], ((m >> 1) - 1) & 1, &abort_s);
      return __shfl_sync(0xffffffffu, okw, 0) != 0;
    };
    for (int t0 = tile0; go && t0 < prm.n_tiles; t0 += 32) {
      const int tt = t0 + lane;
      const bool rel = tt < prm.n_tiles && (tt < tile_own || (__ldg(tm_row + tt) & bsel) != 0);
      // this split's share of the window's relevant tiles
      uint32_t ballot = __ballot_sync(0xffffffffu, rel), mine = 0u;
      while (ballot) {
        const int bit = __ffs(ballot) - 1;
        ballot &= ballot - 1;
        if (ord++ % prm.n_split == split) mine |= 1u << bit;
      }
      while (mine) {
        const int bit = __ffs(mine) - 1;
        mine &= mine - 1;
        const int tt2 = t0 + bit;
        const int pos_t = tt2 * P;
        // the next tile of the window into L2 while this one is loaded: a
        // box with one sector to fetch from DRAM would wait a DRAM round trip
        if (mine && lane == 0) {
          const int pn = (t0 + __ffs(mine) - 1) * P;
#pragma unroll
          for (int kb2 = 0; kb2 < 2; ++kb2) {
            tma_prefetch_l2_3d(&tmQ, kb2 * 64, b * prm.n_q + g * G, pn);
            tma_prefetch_l2_3d(&tmdO, kb2 * 64, b * prm.n_q + g * G, pn);
          }
        }
        const int qs = bwd_qslot(n_it), ds = bwd_dslot(n_it);
        // Q and the row data (the slot freed first)
        if (!take(qs, n_it)) { go = false; break; }
        if (lane == 0) {
          slot_tile[qs] = tt2;
          mbar_arrive_expect_tx(&bar_full[qs], T_BYTES);
#pragma unroll
          for (int kb2 = 0; kb2 < 2; ++kb2)
            tma_load_3d(sT + qs * T_BYTES + kb2 * QBOX, &tmQ, &bar_full[qs], kb2 * 64, b * prm.n_q + g * G, pos_t);
        }
        // lse and D: head h's P positions are contiguous (16-byte pieces)
        Tile* in = tiles + qs;
        for (int e = lane; e < 2 * G * (P / 4); e += 32) {
          const int which = e / (G * (P / 4));
          const int rem = e % (G * (P / 4));
          const int h = rem / (P / 4), q4 = rem % (P / 4);
          const size_t src = ((size_t)b * prm.n_q + g * G + h) * prm.seq + pos_t + q4 * 4;
          cp_async_16((which ? in->D : in->lse) + h * P + q4 * 4, (which ? prm.Drow : prm.lse) + src);
        }
        for (int e = lane; e < P * NCK; e += 32) {
          const int p2 = e / NCK, ck = e % NCK;
          if (kc0 + ck < prm.n_c)                // an odd chunk count leaves a half block
            cp_async_4(&in->w[p2][ck], prm.w + ((size_t)bg * prm.seq + pos_t + p2) * prm.n_c + kc0 + ck);
        }
        for (int p2 = lane; p2 < P; p2 += 32)
          cp_async_4(&in->mword[p2], prm.mask + ((size_t)bg * prm.seq + pos_t + p2) * prm.nw + wsel);
        cp_async_arrive_noinc(&bar_full[qs]);
        n_it = n_it + 1;
        // dO
        if (!take(ds, n_it - 1)) { go = false; break; }
        if (lane == 0) {
          mbar_arrive_expect_tx(&bar_full[ds], T_BYTES);
#pragma unroll
          for (int kb2 = 0; kb2 < 2; ++kb2)
            tma_load_3d(sT + ds * T_BYTES + kb2 * QBOX, &tmdO, &bar_full[ds], kb2 * 64, b * prm.n_q + g * G, pos_t);
        }
        __syncwarp();
        mbar_arrive(&bar_full[ds]);
        n_do = n_it;
      }
    }
    if (go) {
      // end of the walk: the next tile's Q slot carries tile id -1
      const int qs = bwd_qslot(n_it);
      if (take(qs, n_it)) {
        if (lane == 0) {
          slot_tile[qs] = -1;
          mbar_arrive(&bar_full[qs]);
        }
        __syncwarp();
        mbar_arrive(&bar_full[qs]);
      }
    }
    if (abort_s && lane == 0) {
      // copies in flight: K, V and the last two tiles' Q and dO
      mbar_wait(&bar_kv, 0, nullptr);
      for (int j = (n_it > 2 ? n_it - 2 : 0); j < n_it; ++j)
        mbar_wait(&bar_full[bwd_qslot(j)], (j >> 1) & 1, nullptr);
      for (int j = (n_do > 2 ? n_do - 2 : 0); j < n_do; ++j)
        mbar_wait(&bar_full[bwd_dslot(j)], (j >> 1) & 1, nullptr);
    }
    cp_async_wait_all();
  } else if (warp == W_MMA) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idT = idesc_bf16_f32(128, 128, 0, 0);    // S^T, dP^T: keys x rows
    constexpr uint32_t idA = idesc_bf16_f32(128, D, 0, 1);      // dV, dK: keys x d
    const bool leader = elect_one();
    const uint64_t dKk = sw128_desc(smem_u32(sK), 16, 1024);     // K, V as the K-major A
    const uint64_t dVk = sw128_desc(smem_u32(sV), 16, 1024);
    const uint64_t dTk0 = sw128_desc(smem_u32(sT), 16, 1024);    // Q, dO as the K-major B
    const uint64_t dTm0 = sw128_desc(smem_u32(sT), QBOX, 1024);  // Q, dO as the MN-major B
    auto wait_all = [&](uint64_t* bar, uint32_t par) {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, &abort_s));
    };
    // S^T(n) or dP^T(n) from ring slot s
    auto issue_t = [&](uint32_t dst, uint64_t a0, uint64_t b0, int s, uint64_t* bar) {
      if (leader) {
        const uint32_t so = (uint32_t)(s * T_BYTES);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * QBOX + (kk & 3) * 32;
          tc_mma_ss(dst, a0 + (off >> 4), b0 + ((so + off) >> 4), idT, kk > 0 ? 1u : 0u);
        }
        tc_commit(bar);
      }
      __syncwarp();
    };
    // dV or dK += (P^T or dS^T) (dO or Q): K-steps of 16 rows; rows 64 h +
    // 16 j .. of the packed operand sit at columns 64 h + 8 j
    auto issue_a = [&](uint32_t dst, uint32_t a_tm, uint64_t b0, int s, bool first) {
      if (leader) {
        const uint32_t so = (uint32_t)(s * T_BYTES);
#pragma unroll
        for (int kk = 0; kk < 128 / 16; ++kk)
          tc_mma_ts(dst, a_tm + (kk >> 2) * 64 + (kk & 3) * 8, b0 + ((so + kk * 2048) >> 4), idA,
                    (!first || kk > 0) ? 1u : 0u);
      }
    };
    // tile n's Q and row data have landed; false at the end of the walk or on
    // a timeout
    auto next_tile = [&](int n, bool& ok) {
      const int x = bwd_qslot(n);
      if (!(ok = wait_all(&bar_full[x], (n >> 1) & 1))) return false;
      tc_fence_after();
      return slot_tile[x] >= 0;
    };
    // dO of tile n has landed
    auto wait_do = [&](int n) {
      if (!wait_all(&bar_full[bwd_dslot(n)], (n >> 1) & 1)) return false;
      tc_fence_after();
      return true;
    };
    bool ok = wait_all(&bar_kv, 0);
    bool have = ok && next_tile(0, ok);
    if (have) {
      issue_t(tmem + TM_S, dKk, dTk0, bwd_qslot(0), &bar_s_full);
      if (wait_do(0)) issue_t(tmem + TM_DP, dVk, dTk0, bwd_dslot(0), &bar_dp_full);
      else have = ok = false;
    }
    for (int n = 0; have; ++n) {
      if (!(ok = wait_all(&bar_p_full, n & 1))) break;
      tc_fence_after();
      issue_a(tmem + TM_DV, tmem + TM_S, dTm0, bwd_dslot(n), n == 0);
      if (leader) tc_commit(&bar_empty[bwd_dslot(n)]);
      __syncwarp();
      have = next_tile(n + 1, ok);
      if (!ok) break;
      if (have) issue_t(tmem + TM_S, dKk, dTk0, bwd_qslot(n + 1), &bar_s_full);
      if (!(ok = wait_all(&bar_ds_full, n & 1))) break;
      tc_fence_after();
      issue_a(tmem + TM_DK, tmem + TM_DP, dTm0, bwd_qslot(n), n == 0);
      if (leader) tc_commit(&bar_empty[bwd_qslot(n)]);
      __syncwarp();
      if (have) {
        if (!wait_do(n + 1)) {
          ok = false;
          break;
        }
        issue_t(tmem + TM_DP, dVk, dTk0, bwd_dslot(n + 1), &bar_dp_full);
      }
    }
    if (leader) tc_commit(&bar_fin);
    __syncwarp();
    if (abort_s && lane == 0) mbar_wait(&bar_fin, 0, nullptr);
  } else {
    // ------------------------------------------------------------ key threads (warps 0-7)
    const int k = tid & 127;                     // key of the block = TMEM lane
    const int half = warp >> 2;                  // rows 64 half .. 64 half + 63 of a tile
    const int kpos = key0 + k;
    const int kchunk = kpos / CHUNK;
    const int ck = kchunk - kc0;                 // the key's chunk within the block
    const uint32_t tlane = (uint32_t)((warp & 3) * 32) << 16;
    const uint64_t sc2 = f2_pack(prm.scale_log2, prm.scale_log2);
    bool ok = true;
    int n = 0;
    for (;; ++n) {
      // every exit of this loop is taken by all key threads together: the
      // named barrier below is reached once per tile by each of them
      const int s = bwd_qslot(n);
      const bool okw = ok && mbar_wait(&bar_full[s], (n >> 1) & 1, &abort_s);
      const int tt = okw ? slot_tile[s] : -1;
      Tile* in = tiles + s;
      const int pos_t = tt * P;
      const int c_t = pos_t / CHUNK;
      if (tt >= 0 && (tid >> 7) < NCK) {         // one row-table entry per thread
        const int c2 = tid >> 7, t = tid & 127;
        const int pp = t >> prm.lgG, hh = t & (G - 1);
        const int ri = hh * P + pp;
        const float l2 = in->lse[ri] * 1.4426950408889634f;
        const int kch = kc0 + c2;
        float off = -INFINITY;
        if (kch == c_t) off = -l2;
        else if (kch < c_t && ((in->mword[pp] >> (kch & 31)) & 1u))
          off = (prm.sigma != 0.f ? prm.sigma * lg2f(in->w[pp][c2]) : 0.f) - l2;
        in->off[c2][t] = off;
        in->dd[c2][t] = in->D[ri];
      }
      if (!bar_and(1, NKT, okw)) { ok = false; break; }
      if (tt < 0) break;                         // uniform once every wait succeeded
      // causal on the diagonal chunk: row t sees key kpos iff its position
      // pos_t + t / G >= kpos, i.e. t >= (kpos - pos_t) G
      const int colmin = kchunk == c_t ? (kpos - pos_t) * G : 0;
      const float* toff = in->off[ck] + half * 64;
      const float* tdd = in->dd[ck] + half * 64;
      const int cm = colmin - half * 64;         // in this warp's columns
      if (!__all_sync(0xffffffffu, mbar_wait(&bar_s_full, n & 1, &abort_s))) {
        ok = false;
        continue;                                // the next vote ends the walk
      }
      tc_fence_after();
      float pf[64];                              // P of this key and the warp's 64 rows
      {
        float sv[64];
        tmem_ld64(tmem + tlane + TM_S + half * 64, sv);
        // p = 2^(s * scale + off): 3 of every 8 pairs on the FMA pipe
        // (exp2_poly2), the rest on the special-function unit
        constexpr uint32_t kPolyPairs = 0x52u;   // pairs 1, 4, 6 of each 8
        uint32_t pk[32];
        // the causal test only where the tile holds the key's own chunk
        // (warp-uniform: a warp's 32 keys lie in one chunk)
        auto pass = [&](auto causal) {
#pragma unroll
          for (int j2 = 0; j2 < 16; ++j2) {
            const float4 o4 = *reinterpret_cast<const float4*>(toff + 4 * j2);
#pragma unroll
            for (int h2 = 0; h2 < 2; ++h2) {
              const int j = 2 * j2 + h2;
              const uint64_t x = f2_fma(f2_pack(sv[2 * j], sv[2 * j + 1]), sc2,
                                        h2 ? f2_pack(o4.z, o4.w) : f2_pack(o4.x, o4.y));
              float e0, e1;
              if ((kPolyPairs >> (j & 7)) & 1u) {
                exp2_poly2(x, e0, e1);
              } else {
                float x0, x1;
                f2_unpack(x, x0, x1);
                e0 = ex2f(x0);
                e1 = ex2f(x1);
              }
              if (decltype(causal)::value) {
                e0 = 2 * j >= cm ? e0 : 0.f;
                e1 = 2 * j + 1 >= cm ? e1 : 0.f;
              }
              pf[2 * j] = e0;
              pf[2 * j + 1] = e1;
              pk[j] = pack_bf16x2(e0, e1);
            }
          }
        };
        if (cm > 0) pass(std::true_type{});
        else pass(std::false_type{});
        uint32_t h0[16], h1[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          h0[i] = pk[i];
          h1[i] = pk[16 + i];
        }
        tmem_st16u(tmem + tlane + TM_S + half * 64, h0);        // P^T over S^T
        tmem_st16u(tmem + tlane + TM_S + half * 64 + 16, h1);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_p_full);
      if (!__all_sync(0xffffffffu, mbar_wait(&bar_dp_full, n & 1, &abort_s))) {
        ok = false;
        continue;
      }
      tc_fence_after();
      {
        float dp[64];
        tmem_ld64(tmem + tlane + TM_DP + half * 64, dp);
        uint32_t h0[16], h1[16];
#pragma unroll
        for (int j2 = 0; j2 < 16; ++j2) {
          const float4 d4 = *reinterpret_cast<const float4*>(tdd + 4 * j2);
#pragma unroll
          for (int h2 = 0; h2 < 2; ++h2) {
            const int j = 2 * j2 + h2;
            const uint64_t ds = f2_mul(f2_pack(pf[2 * j], pf[2 * j + 1]),
                                       f2_sub(f2_pack(dp[2 * j], dp[2 * j + 1]),
                                              h2 ? f2_pack(d4.z, d4.w) : f2_pack(d4.x, d4.y)));
            float a0, a1;
            f2_unpack(ds, a0, a1);
            (j < 16 ? h0[j] : h1[j - 16]) = pack_bf16x2(a0, a1);
          }
        }
        tmem_st16u(tmem + tlane + TM_DP + half * 64, h0);       // dS^T over dP^T
        tmem_st16u(tmem + tlane + TM_DP + half * 64 + 16, h1);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_ds_full);
    }
    // kpos < seq is warp-uniform (seq is a multiple of 64); warps 0-3 write
    // dK, warps 4-7 dV
    if (ok && __all_sync(0xffffffffu, mbar_wait(&bar_fin, 0, &abort_s)) && kpos < prm.seq) {
      tc_fence_after();
      const bool direct = prm.n_split == 1;
      const float ks = half ? 1.f : (direct ? prm.scale : 1.f);
      float* row;
      if (direct)
        row = (half ? prm.dV : prm.dK) + ((size_t)bg * prm.seq + kpos) * D;
      else
        row = prm.part + (((size_t)split * prm.n_bg + bg) * prm.seq + kpos) * (2 * D) + half * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        float o[32];
        if (n > 0) {
          tmem_ld32(tmem + tlane + (half ? TM_DV : TM_DK) + cc * 32, o);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) o[e] = 0.f;
        }
        float4* dst = reinterpret_cast<float4*>(row + cc * 32);
#pragma unroll
        for (int q4 = 0; q4 < 8; ++q4)
          dst[q4] = make_float4(o[4 * q4] * ks, o[4 * q4 + 1] * ks, o[4 * q4 + 2] * ks, o[4 * q4 + 3] * ks);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == W_MMA) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int CHUNK>
inline size_t attn_bwd_dkv_smem_bytes() {
  return (size_t)2 * 2 * 128 * 128 + (size_t)kBwdDkvSlots * 2 * 128 * 128 +
         kBwdDkvSlots * sizeof(BwdTile<128 / CHUNK>) + 1024;
}

// dK = scale * sum of the splits' partial dK, dV = their sum, in split order.
__global__ void attn_bwd_dkv_reduce_kernel(const float* __restrict__ part, float* __restrict__ dK,
                                           float* __restrict__ dV, long long rows, int n_split, float scale) {
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;   // one float4 of a row
  if (i >= rows * 64) return;
  const long long row = i >> 6;
  const int c4 = (int)(i & 63);                  // 0..31: dK, 32..63: dV
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int s = 0; s < n_split; ++s) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(part + ((size_t)s * rows + row) * 256) + c4);
    acc.x += v.x;
    acc.y += v.y;
    acc.z += v.z;
    acc.w += v.w;
  }
  if (c4 < 32) {
    reinterpret_cast<float4*>(dK + row * 128)[c4] =
        make_float4(acc.x * scale, acc.y * scale, acc.z * scale, acc.w * scale);
  } else {
    reinterpret_cast<float4*>(dV + row * 128)[c4 - 32] = acc;
  }
}

// dQ / dw kernel, then the dK / dV kernel (and, when the key blocks' tile
// lists are split, the reduction of the splits), on one stream: each reads
// what the one before wrote.  K / V maps: boxes of 64 rows (kv64) for the dQ
// kernel, 128 rows (kv128) for the dK / dV kernel.
template <int CHUNK>
cudaError_t launch_attn_bwd_tc(const CUtensorMap& tq, const CUtensorMap& tdo, const CUtensorMap& tk64,
                               const CUtensorMap& tv64, const CUtensorMap& tk128,
                               const CUtensorMap& tv128, const BwdParams& prm, cudaStream_t st) {
  const size_t smem_a = attn_bwd_dq_smem_bytes(prm.n_c, prm.nw, prm.P);
  const size_t smem_b = attn_bwd_dkv_smem_bytes<CHUNK>();
  auto ka = attn_bwd_dq_kernel<CHUNK>;
  auto kb = attn_bwd_dkv_kernel<CHUNK>;
  cudaError_t e = cudaFuncSetAttribute(ka, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_a);
  if (e == cudaSuccess) e = cudaFuncSetAttribute(kb, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_b);
  if (e != cudaSuccess) return e;
  ka<<<(unsigned)(prm.n_tiles * prm.n_bg), 32 * (kBwdRowWarps + 2), smem_a, st>>>(tq, tdo, tk64, tv64, prm);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int n_kb = (prm.seq + 127) / 128;
  kb<<<(unsigned)(n_kb * prm.n_bg * prm.n_split), 32 * (kBwdKeyWarps + 2), smem_b, st>>>(tq, tdo, tk128, tv128,
                                                                                   prm);
  e = cudaGetLastError();
  if (e != cudaSuccess || prm.n_split == 1) return e;
  const long long rows = (long long)prm.n_bg * prm.seq;
  attn_bwd_dkv_reduce_kernel<<<(unsigned)((rows * 64 + 255) / 256), 256, 0, st>>>(
      prm.part, prm.dK, prm.dV, rows, prm.n_split, prm.scale);
  return cudaGetLastError();
}

// Scratch of the kernels: D rows [b, n_q, seq] fp32, the tile unions
// [b * n_kv, nw, seq / P] u32 and, when split, the partial dK | dV rows
// [n_split, b * n_kv * seq, 256] fp32; each part 256-byte aligned.
struct BwdWorkspace {
  size_t d_off, t_off, p_off, total;
  int n_split;
};

inline BwdWorkspace attn_bwd_tc_workspace(int batch, int n_q, int n_kv, int seq, int n_c) {
  const int G = n_q / n_kv, P = 128 / G;
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  BwdWorkspace w;
  w.n_split = attn_bwd_n_split((seq + 127) / 128, batch * n_kv);
  w.d_off = 0;
  w.t_off = up((size_t)batch * n_q * seq * 4);
  w.p_off = w.t_off + up((size_t)batch * n_kv * ((n_c + 31) / 32) * (seq / P) * 4);
  w.total = w.p_off + (w.n_split > 1 ? up((size_t)w.n_split * batch * n_kv * seq * 256 * 4) : 0);
  return w;
}

}  // namespace dash
