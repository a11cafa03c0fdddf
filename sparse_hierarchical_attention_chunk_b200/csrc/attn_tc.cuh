// Stage 2 (bf16): prior-induced block-sparse softmax attention on tcgen05.
//
// gist.science technical summary, "Fase 2: Prior-Geinduceerde Spaarzame
// Softmax": softmax seen as the maximiser of z^T p - KL(p || u) with the
// reference u replaced by a prior g from the routing weights w, g = 0 where
// w = 0 (masked chunks), a separate branch for the chunk on the diagonal,
// and a FlashAttention-style kernel that walks the active chunks of a
// bit-packed mask and adds the routing bias to the logits before the softmax.
// With g = w_b^sigma per key of routed block b and 1 on the query's own
// chunk: p_ij ~ exp(q.k/sqrt(d) + sigma ln w_ib), i.e. a bias added to S.
//
// Work unit.  A CTA owns two tiles of M = 128 query rows each.  A tile is
// all G query heads of one KV head at P = 128 / G consecutive positions,
// rows ordered position-major (r = p * G + h), so the G heads of a position
// -- which share one routing support -- sit in adjacent TMEM lanes.  The two
// tiles are consecutive position ranges of one chunk; the CTA walks the
// union of their routed chunks plus the diagonal chunk (first, so every row
// starts with a finite running max).  K/V blocks are loaded once for both.
//
// Per block, per tile: the tile's MMAs are skipped when none of its rows
// routes to the block; inside an active tile, a warp whose 32 rows are all
// inactive skips the softmax and only clears its P rows.
//
// Roles (320 threads):
//   warps 0-3 / 4-7  softmax of tile 0 / tile 1: thread = row = TMEM lane.
//              S row from TMEM, bias, online softmax with a lazy rescale (O
//              in TMEM corrected only when the row max grows by more than
//              2^8), P written back as bf16 over S in TMEM, epilogue O/l.
//   warp 8     TMA producer: Q tiles once (3-D boxes {64, G, P}); K, V blocks
//              (2-D boxes {64, B}) into NS-stage rings with separate
//              full/empty barriers for K and V.
//   warp 9     TMEM allocation (all 512 columns) and tcgen05.mma issue:
//              S = Q K^T (SS: both from shared memory, M=128, N=B, K=d) and
//              O += P V (TS: P from TMEM, V from shared memory, MN-major,
//              M=128, N=d, K=B).  With B = 64 each tile has two S buffers and
//              S of block j+2 is issued right after PV of block j; with
//              B = 128 one buffer, S of block j+1 after PV of block j.  While
//              one tile's softmax runs, the tensor core works on the other.
// All waits are bounded (mbarrier try_wait + globaltimer); on a timeout
// every role unwinds, copies in flight are awaited and TMEM is released.
#pragma once

#include <cuda.h>
#include "dash_common.cuh"
#include "tmem_wide.cuh"

namespace dash {

struct AttnParams {
  // w: dense [rows][n_c], or (packed != 0) the compact form of stage 1:
  // per row the weights of its routed chunks in increasing chunk order
  const float* w;
  const uint32_t* mask;
  int packed;
  __nv_bfloat16* O;
  float* lse;
  int n_q, n_kv, seq, chunk, n_c, nw, G, P, n_ctiles, n_bg;
  float sigma, scale_log2;
};

// D[tmem] (+)= A[tmem] * B[smem desc]^T, kind::f16 (bf16 in, fp32 acc).
__device__ __forceinline__ void tc_mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_st16u(uint32_t taddr, const uint32_t (&v)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]),
        "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]),
        "r"(v[14]), "r"(v[15])
      : "memory");
}

// ---------------------------------------------------------------------------
// softmax arithmetic helpers
// ---------------------------------------------------------------------------
// (f2_* pair arithmetic and fmax3 live in dash_common.cuh)

// 2^x for a pair, on the FMA pipe instead of the special-function unit
// (which is the softmax bottleneck: 16 results per clock per SM against the
// 8192 exponentials a 128 x 64 S tile needs per 262 tensor-core clocks).
// x = n + f with n = round(x) taken from the low mantissa bits of
// x + 1.5 * 2^23; 2^f for f in [-1/2, 1/2] from a degree-3 polynomial fitted
// for minimum maximum relative error (7.5e-5, by iteratively reweighted
// least squares; far below the 2^-9 rounding of the bf16 P it feeds); 2^n is
// added to the exponent field with an integer multiply-add.  Inputs are
// clamped at -125 so the exponent cannot wrap: -inf gives ~2^-125, which is
// negligible next to the row maximum of 1.
__device__ __forceinline__ void exp2_poly2(uint64_t x, float& e0, float& e1) {
  constexpr float kMagic = 12582912.f;             // 1.5 * 2^23
  float x0, x1;
  f2_unpack(x, x0, x1);
  x = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t M = f2_pack(kMagic, kMagic);
  const uint64_t t = f2_add(x, M);
  const uint64_t fr = f2_sub(x, f2_sub(t, M));    // in [-1/2, 1/2]
  uint64_t p = f2_fma(fr, f2_pack(0.055171665f, 0.055171665f), f2_pack(0.24261117f, 0.24261117f));
  p = f2_fma(p, fr, f2_pack(0.69326097f, 0.69326097f));
  p = f2_fma(p, fr, f2_pack(0.99992806f, 0.99992806f));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  e0 = __int_as_float(__float_as_int(t0) * 8388608 + __float_as_int(p0));
  e1 = __int_as_float(__float_as_int(t1) * 8388608 + __float_as_int(p1));
}

// Key blocks of BLK keys, one chunk each (BLK = B = 64 or 128).
template <int BLK, int D>
struct TcLayout {
  static_assert(BLK == 64 || BLK == 128, "64- or 128-key blocks");
  static constexpr int NT = 2;                      // tiles per CTA
  static constexpr int NS = BLK == 64 ? 3 : 2;      // K and V ring depth
  // With 64-key blocks Q is copied into TMEM and S = Q K^T runs as a
  // TS-MMA, so the tensor core reads only K from shared memory (with Q from
  // shared memory too, an N = 64 MMA needs more shared-memory bandwidth than
  // there is).  With 128-key blocks S takes 128 TMEM columns per tile, which
  // leaves no room for Q: S runs as an SS-MMA with N = 128 (half the
  // shared-memory bytes per FLOP of N = 64), and each block step carries
  // twice the MMA work for the same fixed per-step cost of the issuing warp.
  static constexpr bool QTM = BLK == 64;
  static constexpr int QBOX = 128 * 128;            // 128 rows x 128 B (64 bf16 columns)
  static constexpr int Q_BYTES = QBOX * (D / 64);   // one tile
  static constexpr int KV_BOX = BLK * 128;          // BLK rows x 128 B
  static constexpr int KV_BYTES = KV_BOX * (D / 64);
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + NT * Q_BYTES;
  static constexpr int OFF_V = OFF_K + NS * KV_BYTES;
  static constexpr int OFF_AUX = OFF_V + NS * KV_BYTES;   // list, codes, mask rows, w ring
  // TMEM columns per tile: [Q as bf16 pairs (QTM only) | S (BLK fp32; P
  // overwrites its first BLK/2 columns as bf16 pairs) | O (D fp32)]
  static constexpr int TM_Q = 0;
  static constexpr int TM_S = QTM ? D / 2 : 0;
  static constexpr int TM_O = TM_S + BLK;
  static constexpr int TM_TILE = TM_O + D;
  static constexpr int TM_COLS = 512;
  static_assert(NT * TM_TILE <= TM_COLS, "TMEM budget");
};

// 320 threads, one CTA per SM: ten warps put three on some of the SM's four
// sub-partitions, whose 16 K registers then allow 168 per thread.
template <int CHUNK, int D>
__global__ void __launch_bounds__(320, 1) attn_fwd_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
    const __grid_constant__ CUtensorMap tmV, const AttnParams prm) {
  constexpr int BLK = CHUNK;                     // keys per MMA block: one chunk
  constexpr int SB = CHUNK / BLK;                // sub-blocks per chunk (1)
  using L = TcLayout<BLK, D>;
  constexpr int NS = L::NS;
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned by pointer arithmetic on the shared array, so that the
  // compiler keeps the shared address space (and emits shared loads)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  int* list = reinterpret_cast<int*>(smem + L::OFF_AUX);             // [n_c + 1]
  uint8_t* code = reinterpret_cast<uint8_t*>(list + prm.n_c + 1);    // [n_c + 1], bit t: tile t active
  uint8_t* code_end = code + prm.n_c + 1;                          // rounded up to 16 bytes
  uint32_t* mrows = reinterpret_cast<uint32_t*>(code_end + ((16u - (smem_u32(code_end) & 15u)) & 15u));
  // compact weights: set bits of each position's mask before each word
  int* mpre = reinterpret_cast<int*>(mrows + 2 * prm.P * prm.nw);          // [2P][nw]
  float* w_sm = reinterpret_cast<float*>(mpre + 2 * prm.P * prm.nw);       // [NS][2P]
  const int n_wl = min(2 * prm.P, 32);      // producer lanes that fetch w

  // Barriers.  Each tile has one S buffer, so every barrier below advances at
  // most one phase ahead of its waiter: s_full[t] (S of tile t ready; its
  // completion also implies every earlier PV of the tile is done), p_full[t]
  // (P of tile t written, 128 softmax arrivals), o_done[t] (a PV of tile t
  // done), fin[t] (once: the last PV of tile t done), q_tm (Q copied into
  // TMEM, 256 arrivals), K/V ring full/empty pairs.
  __shared__ __align__(8) uint64_t bar_q, bar_q_tm;
  __shared__ __align__(8) uint64_t bar_s_full[2], bar_p_full[2], bar_o_done[2], bar_fin[2];
  __shared__ __align__(8) uint64_t bar_k_full[NS], bar_k_empty[NS], bar_v_full[NS], bar_v_empty[NS];
  __shared__ uint32_t tmem_slot;
  __shared__ int nb_s, cnt_s[2];
  __shared__ volatile int abort_s;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // (b, h_kv)-major, late (heavy) tiles first: the CTAs resident at any one
  // time share one K/V head, whose blocks then stay in L2 across tiles
  const int ctile = prm.n_ctiles - 1 - (int)(blockIdx.x % prm.n_ctiles);
  const int bg = (int)(blockIdx.x / prm.n_ctiles);
  const int b = bg / prm.n_kv, g = bg % prm.n_kv;
  const int P = prm.P, G = prm.G;
  const int pos0 = ctile * 2 * P;
  const int c_i = pos0 / prm.chunk;

  if (warp == 9) {
    tmem_alloc(&tmem_slot, L::TM_COLS);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_q, 1);
    mbar_init(&bar_q_tm, 256);
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar_s_full[t], 1);
      mbar_init(&bar_p_full[t], 128);
      mbar_init(&bar_o_done[t], 1);
      mbar_init(&bar_fin[t], 1);
    }
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar_k_full[s], 1);
      mbar_init(&bar_k_empty[s], 1);
      mbar_init(&bar_v_full[s], 1 + n_wl);   // TMA tx arrival + one per w-fetching lane
      mbar_init(&bar_v_empty[s], 1);
    }
    abort_s = 0;
    fence_mbar_init();
  }
  if (tid == 256) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  // routing masks of the CTA's 2P positions
  const size_t row0 = (size_t)bg * prm.seq + pos0;
  for (int i = tid; i < 2 * P * prm.nw; i += blockDim.x) mrows[i] = prm.mask[row0 * prm.nw + i];
  __syncthreads();
  // block list: the diagonal chunk, then the union of routed chunks c < c_i,
  // each with a 2-bit code of the tiles that route to it
  if (warp == 0) {
    int base = 1, cnt0 = 0, cnt1 = 0;
    for (int k0 = 0; k0 < prm.nw; k0 += 32) {
      const int k = k0 + lane;
      uint32_t u0 = 0, u1 = 0;
      if (k < prm.nw && k * 32 < c_i) {
        for (int p = 0; p < P; ++p) {
          u0 |= mrows[p * prm.nw + k];
          u1 |= mrows[(P + p) * prm.nw + k];
        }
        const int rem = c_i - k * 32;
        if (rem < 32) {
          u0 &= (1u << rem) - 1u;
          u1 &= (1u << rem) - 1u;
        }
      }
      cnt0 += __popc(u0);
      cnt1 += __popc(u1);
      uint32_t u = u0 | u1;
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
        list[at] = k * 32 + bit;
        code[at] = (uint8_t)(((u0 >> bit) & 1u) | (((u1 >> bit) & 1u) << 1));
        ++at;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
    cnt0 = __reduce_add_sync(0xffffffffu, cnt0);
    cnt1 = __reduce_add_sync(0xffffffffu, cnt1);
    if (lane == 0) {
      list[0] = c_i;
      code[0] = 3;
      nb_s = base;
      cnt_s[0] = cnt0;
      cnt_s[1] = cnt1;
    }
  }
  if (prm.packed && warp >= 1 && warp < 8) {
    // the rank of chunk c in position q's compact row is mpre[q][c / 32]
    // plus the set bits of word c / 32 below c
    for (int q = tid - 32; q < 2 * P; q += 224) {
      int acc = 0;
      for (int k = 0; k < prm.nw; ++k) {
        mpre[q * prm.nw + k] = acc;
        acc += __popc(mrows[q * prm.nw + k]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  const int nb = nb_s;
  // Sub-block sequence: the diagonal chunk's sub-blocks first (its second
  // 64-key half only for tiles with a position that reaches it), then SB
  // sub-blocks per routed chunk.  Every role walks it with entry().
  const int diag_lo = c_i * CHUNK;
  int dcode1 = 0;                              // tiles active on diagonal sub-block 1
  if (SB == 2) {
    if (pos0 + P - 1 >= diag_lo + BLK) dcode1 |= 1;
    if (pos0 + 2 * P - 1 >= diag_lo + BLK) dcode1 |= 2;
  }
  const int n_diag = 1 + (dcode1 != 0);
  const int nbb = n_diag + (nb - 1) * SB;     // sub-blocks walked by the CTA
  const int nblk_t[2] = {cnt_s[0] * SB + 1 + (dcode1 & 1), cnt_s[1] * SB + 1 + ((dcode1 >> 1) & 1)};
  struct Entry { int j, c, sb, code; };
  auto entry = [&](int jj) {
    Entry e;
    if (jj < n_diag) {
      e.j = 0; e.c = c_i; e.sb = jj; e.code = jj == 0 ? 3 : dcode1;
    } else {
      const int r = jj - n_diag;
      e.j = 1 + r / SB; e.sb = r % SB; e.c = list[e.j]; e.code = code[e.j];
    }
    return e;
  };

  uint8_t* sQ = smem + L::OFF_Q;
  uint8_t* sK = smem + L::OFF_K;
  uint8_t* sV = smem + L::OFF_V;

  if (warp == 8) {
    // ------------------------------------------------------------ producer
    // lane 0 issues the TMA copies; lanes < n_wl also fetch, with cp.async,
    // the routing weight w[position, chunk] of the block for the CTA's 2P
    // positions into w_sm, completing on the same barrier as the V tile.
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar_q, 2 * L::Q_BYTES);
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_3d(sQ + t * L::Q_BYTES + kb * L::QBOX, &tmQ, &bar_q, kb * 64,
                      b * prm.n_q + g * G, pos0 + t * P);
    }
    int issued_k = 0, issued_v = 0;
    for (int j = 0; j < nbb; ++j) {            // j: sub-block index
      const int s = j % NS;
      const uint32_t par = ((j / NS) & 1) ^ 1;
      const Entry en = entry(j);
      const int c = en.c;
      const int krow = bg * prm.seq + c * CHUNK + en.sb * BLK;
      int okw = lane == 0 ? (int)mbar_wait(&bar_k_empty[s], par, &abort_s) : 0;
      if (!__shfl_sync(0xffffffffu, okw, 0)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar_k_full[s], L::KV_BYTES);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_2d(sK + s * L::KV_BYTES + kb * L::KV_BOX, &tmK, &bar_k_full[s], kb * 64, krow);
      }
      issued_k = j + 1;
      okw = lane == 0 ? (int)mbar_wait(&bar_v_empty[s], par, &abort_s) : 0;
      if (!__shfl_sync(0xffffffffu, okw, 0)) break;
      if (lane == 0) {
        mbar_arrive_expect_tx(&bar_v_full[s], L::KV_BYTES);
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb)
          tma_load_2d(sV + s * L::KV_BYTES + kb * L::KV_BOX, &tmV, &bar_v_full[s], kb * 64, krow);
      }
      if (lane < n_wl) {
        for (int q = lane; q < 2 * P; q += 32) {
          // a position that does not route to c reads a neighbouring entry
          // of its own row (never used: its bias is -inf)
          const int col = prm.packed ? mpre[q * prm.nw + (c >> 5)] +
                                           __popc(mrows[q * prm.nw + (c >> 5)] & ((1u << (c & 31)) - 1u))
                                     : c;
          cp_async_4(w_sm + s * 2 * P + q, prm.w + (row0 + q) * prm.n_c + col);
        }
        cp_async_arrive_noinc(&bar_v_full[s]);
      }
      issued_v = j + 1;
    }
    if (abort_s) {
      // let copies still in flight land before the CTA can exit
      if (lane == 0) {
        for (int j = (issued_k > NS ? issued_k - NS : 0); j < issued_k; ++j)
          mbar_wait(&bar_k_full[j % NS], (j / NS) & 1, nullptr);
        for (int j = (issued_v > NS ? issued_v - NS : 0); j < issued_v; ++j)
          mbar_wait(&bar_v_full[j % NS], (j / NS) & 1, nullptr);
      }
      cp_async_wait_all();
    }
  } else if (warp == 9) {
    // ------------------------------------------------------------ MMA issuer
    // The whole warp runs the issue loop with warp-uniform values (so the
    // descriptor arithmetic stays on the uniform datapath); one elected lane
    // issues each tcgen05 instruction.  Every lane waits on the barriers
    // itself and the loop control is kept uniform with __all_sync.
    // Per block j: PV_0(j), S_0(j+1), PV_1(j), S_1(j+1) -- while one tile's
    // softmax runs, the tensor core works on the other tile.
    constexpr uint32_t idS = idesc_bf16_f32(128, BLK, 0, 0);
    constexpr uint32_t idO = idesc_bf16_f32(128, D, 0, 1);
    const bool leader = elect_one();
    // descriptors: base + (byte offset >> 4) advances the start-address field
    const uint64_t dQ0 = sw128_desc(smem_u32(sQ), 16, 1024);
    const uint64_t dK0 = sw128_desc(smem_u32(sK), 16, 1024);
    const uint64_t dV0 = sw128_desc(smem_u32(sV), L::KV_BOX, 1024);
    int nS0 = 0, nS1 = 0, nP0 = 0, nP1 = 0;    // per-tile S issued / PV issued
    const int nb0 = nblk_t[0], nb1 = nblk_t[1]; // per-tile active sub-blocks
    auto wait_all = [&](uint64_t* bar, uint32_t par) {
      return __all_sync(0xffffffffu, mbar_wait(bar, par, &abort_s));
    };
    auto issue_S = [&](int t, int j) {         // S of tile t for block j (K(j) loaded)
      const int s = j % NS;
      const uint32_t dst = tmem + t * L::TM_TILE + L::TM_S;
      const uint64_t dk = dK0 + (uint64_t)((s * L::KV_BYTES) >> 4);
      if (leader) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t offk = (kk >> 2) * L::KV_BOX + (kk & 3) * 32;
          if constexpr (L::QTM) {
            tc_mma_ts(dst, tmem + t * L::TM_TILE + L::TM_Q + kk * 8, dk + (offk >> 4), idS,
                      kk > 0 ? 1u : 0u);
          } else {
            const uint32_t off = t * L::Q_BYTES + (kk >> 2) * L::QBOX + (kk & 3) * 32;
            tc_mma_ss(dst, dQ0 + (off >> 4), dk + (offk >> 4), idS, kk > 0 ? 1u : 0u);
          }
        }
        tc_commit(&bar_s_full[t]);
      }
      __syncwarp();
      if (t) ++nS1; else ++nS0;
    };
    (void)dQ0;
    bool ok = L::QTM ? wait_all(&bar_q_tm, 0) : wait_all(&bar_q, 0);
    ok = ok && wait_all(&bar_k_full[0], 0);
    if (ok) {
      tc_fence_after();
      issue_S(0, 0);
      issue_S(1, 0);
      if (leader) tc_commit(&bar_k_empty[0]);
      __syncwarp();
    }
    for (int j = 0; ok && j < nbb; ++j) {      // j: sub-block index
      const int s = j % NS;
      const int cj = entry(j).code;
      const int cn = j + 1 < nbb ? entry(j + 1).code : 0;
      if (!(ok = wait_all(&bar_v_full[s], (j / NS) & 1))) break;
      if (cn && !(ok = wait_all(&bar_k_full[(j + 1) % NS], ((j + 1) / NS) & 1))) break;
      const uint64_t dv = dV0 + (uint64_t)((s * L::KV_BYTES) >> 4);
#pragma unroll
      for (int t = 0; t < 2; ++t) {
        if ((cj >> t) & 1) {
          const int idx = t ? nP1 : nP0;
          if (!(ok = wait_all(&bar_p_full[t], idx & 1))) break;
          tc_fence_after();
          const uint32_t pa = tmem + t * L::TM_TILE + L::TM_S;
          const uint32_t od = tmem + t * L::TM_TILE + L::TM_O;
          if (leader) {
#pragma unroll
            for (int kk = 0; kk < BLK / 16; ++kk)
              tc_mma_ts(od, pa + kk * 8, dv + (uint64_t)((kk * 2048) >> 4), idO,
                        (idx > 0 || kk > 0) ? 1u : 0u);
            tc_commit(&bar_o_done[t]);
            if (idx + 1 == (t ? nb1 : nb0)) tc_commit(&bar_fin[t]);
          }
          __syncwarp();
          if (t) ++nP1; else ++nP0;
        }
        // the tile's S buffer is free once its last PV is issued (in order)
        if ((cn >> t) & 1) issue_S(t, j + 1);
      }
      if (!ok) break;
      if (leader) {
        tc_commit(&bar_v_empty[s]);
        if (cn) tc_commit(&bar_k_empty[(j + 1) % NS]);
      }
      __syncwarp();
    }
    if (abort_s && lane == 0) {
      // wait (bounded) for the MMAs already issued before TMEM is freed
      if (nP0 > 0) mbar_wait(&bar_o_done[0], (nP0 - 1) & 1, nullptr);
      if (nP1 > 0) mbar_wait(&bar_o_done[1], (nP1 - 1) & 1, nullptr);
      if (nS0 > 0) mbar_wait(&bar_s_full[0], (nS0 - 1) & 1, nullptr);
      if (nS1 > 0) mbar_wait(&bar_s_full[1], (nS1 - 1) & 1, nullptr);
    }
  } else {
    // ------------------------------------------------------------ softmax (rows)
    const int t = warp >> 2;                  // tile
    const int r = tid & 127;                  // row in the tile = TMEM lane
    const int p = r / G, hq = r % G;
    const int pl = t * P + p;                 // position index within the CTA
    const int pos = pos0 + pl;
    const int qh = g * G + hq;
    const uint32_t tlane = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tT = tmem + tlane + t * L::TM_TILE;
    const uint32_t tS = tT + L::TM_S;
    const uint32_t tO = tT + L::TM_O;
    const uint32_t* mrow = mrows + pl * prm.nw;
    const float scale = prm.scale_log2;
    const float sigma = prm.sigma;
    float m = -INFINITY, l = 0.f;
    int n = 0;                                // blocks of this tile processed
    bool ok = mbar_wait(&bar_q, 0, &abort_s);
    if constexpr (L::QTM) {
      // Q row r of this tile: shared memory (TMA, 128-byte swizzle) -> TMEM as
      // bf16 pairs, the A operand of S = Q K^T
      if (ok) {
        const uint8_t* qrow = sQ + t * L::Q_BYTES + (r >> 3) * 1024 + (r & 7) * 128;
#pragma unroll
        for (int kb = 0; kb < D / 64; ++kb) {
          uint32_t v[32];
#pragma unroll
          for (int ch = 0; ch < 8; ++ch) {
            const uint4 q4 = *reinterpret_cast<const uint4*>(qrow + kb * L::QBOX + ((ch ^ (r & 7)) << 4));
            v[ch * 4 + 0] = q4.x;
            v[ch * 4 + 1] = q4.y;
            v[ch * 4 + 2] = q4.z;
            v[ch * 4 + 3] = q4.w;
          }
          uint32_t h0[16], h1[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            h0[i] = v[i];
            h1[i] = v[16 + i];
          }
          tmem_st16u(tT + L::TM_Q + kb * 32, h0);
          tmem_st16u(tT + L::TM_Q + kb * 32 + 16, h1);
        }
        tmem_wait_st();
      }
      tc_fence_before();
      mbar_arrive(&bar_q_tm);
    }
    for (int jj = 0; ok && jj < nbb; ++jj) {  // jj: sub-block index
      const Entry en = entry(jj);
      if (!((en.code >> t) & 1)) continue;
      const int j = en.j;                     // chunk index in the list (0 = diagonal)
      const int c = en.c;
      const bool act = j == 0 || ((mrow[c >> 5] >> (c & 31)) & 1u);
      if (!mbar_wait(&bar_s_full[t], n & 1, &abort_s)) { ok = false; break; }
      tc_fence_after();
      float bias = 0.f;
      if (j > 0) {
        if (!act) {
          bias = -INFINITY;
        } else if (sigma != 0.f) {
          // w of this block arrived with its V tile (the slot is released only
          // after this tile's P has been consumed)
          if (!mbar_wait(&bar_v_full[jj % NS], (jj / NS) & 1, &abort_s)) { ok = false; break; }
          bias = sigma * lg2f(w_sm[(jj % NS) * 2 * P + pl]);
        }
      }
      if (!__any_sync(0xffffffffu, act)) {
        // no row of this warp routes here: P rows must read as zeros
        uint32_t z[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) z[i] = 0u;
#pragma unroll
        for (int cc = 0; cc < BLK / 32; ++cc) tmem_st16u(tS + cc * 16, z);
      } else {
        // the block's S row in halves of 64 columns (one half for 64-key
        // blocks, which stays in registers; two for 128-key blocks, read
        // once for the max and once for the exponentials)
        constexpr int NH = BLK / 64;
        const int lim = j == 0 ? pos - (c * CHUNK + en.sb * BLK) : BLK;   // causal: keys k <= lim
        float sv[64];
        auto load_half = [&](int hh) {
          tmem_ld64(tS + hh * 64, sv);
          if (j == 0) {
#pragma unroll
            for (int k = 0; k < 64; ++k) sv[k] = hh * 64 + k <= lim ? sv[k] : -INFINITY;
          }
        };
        float mrow = -INFINITY;
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
          load_half(hh);
          // row max: 8 independent partial maxima, three inputs per instruction
          float mp[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) mp[i] = sv[i];
#pragma unroll
          for (int k = 8; k < 64; k += 16)
#pragma unroll
            for (int i = 0; i < 8; ++i) mp[i] = fmax3(mp[i], sv[k + i], k + 8 + i < 64 ? sv[k + 8 + i] : sv[i]);
#pragma unroll
          for (int s2 = 4; s2 > 0; s2 >>= 1)
#pragma unroll
            for (int i = 0; i < s2; ++i) mp[i] = fmaxf(mp[i], mp[i + s2]);
          mrow = fmaxf(mrow, mp[0]);
        }
        const float mx = fmaf(mrow, scale, bias);   // scale > 0: max commutes
        // the first sub-block (diagonal, keys from the chunk start) always has a
        // visible key, so it sets a finite running max
        const float m_new = (jj == 0 || mx > m + 8.f) ? mx : m;
        const float off = bias - m_new;
        // p = 2^(s * scale + off): 3 of every 8 pairs on the FMA pipe
        // (exp2_poly2), the rest on the special-function unit, which balances
        // the unit's 16 results per clock against the issue slots the
        // polynomial takes
        constexpr uint32_t kPolyPairs = 0x52u;          // pairs 1, 4, 6 of each 8
        const uint64_t sc2 = f2_pack(scale, scale), off2 = f2_pack(off, off);
        uint64_t rp[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) rp[i] = 0ull;
        uint32_t pk[32];
        // P of half hh as bf16 pairs, over S columns already read
        auto store_p = [&](int hh) {
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t v[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) v[i] = pk[cc * 16 + i];
            tmem_st16u(tS + hh * 32 + cc * 16, v);
          }
        };
#pragma unroll
        for (int hh = 0; hh < NH; ++hh) {
          if (NH > 1) load_half(hh);
#pragma unroll
          for (int k2 = 0; k2 < 32; ++k2) {
            const uint64_t x = f2_fma(f2_pack(sv[2 * k2], sv[2 * k2 + 1]), sc2, off2);
            float e0, e1;
            if (kPolyPairs & (1u << (k2 & 7))) {
              exp2_poly2(x, e0, e1);
            } else {
              float x0, x1;
              f2_unpack(x, x0, x1);
              e0 = ex2f(x0);
              e1 = ex2f(x1);
            }
            rp[k2 & 3] = f2_add(rp[k2 & 3], f2_pack(e0, e1));
            pk[k2] = pack_bf16x2(e0, e1);
          }
          // a 128-key block writes its first half's P now (its S columns
          // are read), a 64-key block after the rescale below
          if (NH > 1) store_p(hh);
        }
        rp[0] = f2_add(f2_add(rp[0], rp[1]), f2_add(rp[2], rp[3]));
        float rs0, rs1;
        f2_unpack(rp[0], rs0, rs1);
        const float rs = rs0 + rs1;
        if (jj > 0) {
          const bool need = m_new != m;
          if (__any_sync(0xffffffffu, need)) {
            // O must hold every PV issued so far before it is rescaled (the
            // S completion just waited for already implies it)
            if (!mbar_wait(&bar_o_done[t], (n - 1) & 1, &abort_s)) { ok = false; break; }
            tc_fence_after();
            const float corr = need ? ex2f(m - m_new) : 1.f;
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              float o[32];
              tmem_ld32(tO + cc * 32, o);
              float lo[16], hi[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                lo[i] = o[i] * corr;
                hi[i] = o[16 + i] * corr;
              }
              tmem_st16(tO + cc * 32, lo);
              tmem_st16(tO + cc * 32 + 16, hi);
            }
            l *= corr;
          }
        }
        m = m_new;
        l += rs;
        if (NH == 1) store_p(0);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_p_full[t]);
      ++n;
    }
    if (ok && mbar_wait(&bar_fin[t], 0, &abort_s)) {
      tc_fence_after();
      const float inv = 1.f / l;
      __nv_bfloat16* orow = prm.O + (((size_t)b * prm.n_q + qh) * prm.seq + pos) * D;
#pragma unroll
      for (int cc = 0; cc < D / 32; ++cc) {
        float o[32];
        tmem_ld32(tO + cc * 32, o);
        uint4* dst = reinterpret_cast<uint4*>(orow + cc * 32);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint4 v;
          v.x = pack_bf16x2(o[q4 * 8 + 0] * inv, o[q4 * 8 + 1] * inv);
          v.y = pack_bf16x2(o[q4 * 8 + 2] * inv, o[q4 * 8 + 3] * inv);
          v.z = pack_bf16x2(o[q4 * 8 + 4] * inv, o[q4 * 8 + 5] * inv);
          v.w = pack_bf16x2(o[q4 * 8 + 6] * inv, o[q4 * 8 + 7] * inv);
          dst[q4] = v;
        }
      }
      if (prm.lse)
        prm.lse[((size_t)b * prm.n_q + qh) * prm.seq + pos] = (m + log2f(l)) * 0.69314718055994531f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TM_COLS);
  }
}

template <int BLK, int D>
size_t attn_tc_smem_bytes(int n_c, int nw, int P) {
  using L = TcLayout<BLK, D>;
  return (size_t)L::OFF_AUX + (size_t)(n_c + 1) * 5 + 16 + (size_t)2 * P * nw * 8 +
         (size_t)L::NS * 2 * P * 4 + 1024;
}

// CHUNK = 64 or 128 (one key block per chunk), D = 64 or 128; K/V tensor
// maps use {64, CHUNK} boxes.
template <int CHUNK, int D>
cudaError_t launch_attn_tc(const CUtensorMap& tmQ, const CUtensorMap& tmK, const CUtensorMap& tmV,
                           const AttnParams& prm, cudaStream_t st) {
  auto kern = attn_fwd_tc_kernel<CHUNK, D>;
  size_t smem = attn_tc_smem_bytes<CHUNK, D>(prm.n_c, prm.nw, prm.P);
  // every CTA holds all 512 TMEM columns, so it must be alone on its SM:
  // ask for more than half of the shared memory
  if (smem < 118 * 1024) smem = 118 * 1024;
  if (smem > 227 * 1024) return cudaErrorInvalidValue;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  const unsigned grid = (unsigned)(prm.n_ctiles * prm.n_bg);
  kern<<<grid, 320, smem, st>>>(tmQ, tmK, tmV, prm);
  return cudaGetLastError();
}

}  // namespace dash
