// Stage 1 on the tensor core: routing for GQA groups of 16 query heads.
//
// Same operation as route.cuh (gist.science technical summary, "Fase 1: Entmax
// Chunk Routering": logits against the chunk summaries, w = alpha-entmax(gamma
// z), GQA mean over the query heads of a KV head, mask = w > 0), organised
// around tensor memory so that every logit is computed once and read by the
// one thread that owns its row:
//
//  * A CTA owns NPOS consecutive positions of one (b, h_kv) -- all inside one
//    chunk, so they share the eligible chunks c < c_i -- i.e. R = 16 * NPOS
//    rows (position-major, r = p * 16 + h).  The Q tile (TMA, 3-D box) and
//    the chunk summaries Kbar (TMA, 256 chunks per tile) feed tcgen05 MMAs
//    (M = R, N = 256, K = 128) whose fp32 logits land in TMEM: one TMEM lane
//    per row, one column per chunk.
//      Positions whose eligible chunks fit TMEM (c_i <= 512): 8 positions,
//      R = 128, chunk c in column c.
//      Positions with 512 < c_i <= 1024: 4 positions (64 rows) and a K = 256
//      product A_ext B_ext^T with A_ext = [[Q, 0], [0, Q]] and the two
//      128-wide K halves of B_ext taken from chunks n and 512 + n: rows
//      0-63 receive chunks [0, 512) and rows 64-127 chunks [512, 1024) in
//      the same 512 columns.  A row's two halves live in threads m and
//      m + 64, which merge their partial sums through shared memory.
//  * Two threads per row (warps w and w + 4 read the same TMEM lanes, each
//    half of the row's 32-chunk blocks; their partial sums meet in shared
//    memory): the entmax threshold is found with passes over the row's TMEM
//    columns (32 per tcgen05.ld): row max, then Newton from tau = max - 1 on
//    h(tau) = ||[x - tau]_+||_e - 1 (convex, decreasing, nearly linear -> a
//    few steps), then for alpha = 1.5 / 2 the exact root on the support
//    found, kept only if the support is self-consistent.
//  * GQA mean: the 16 heads of a position are 16 adjacent lanes; a 4-step
//    reduce-scatter over them leaves lane h with the sums for chunks
//    c0 + 2h and c0 + 2h + 1 of each 32-chunk block, stored as one float2
//    (the half-warp writes 128 contiguous bytes); the mask word is the OR of
//    the lanes' 2-bit contributions.
#pragma once

#include <cuda.h>
#include "dash_common.cuh"
#include "route.cuh"
#include "tmap.cuh"
#include "tmem_wide.cuh"

namespace dash {

struct RouteTcParams {
  float* w;
  uint32_t* mask;
  // estimate_diagonal: keys and learned queries of stage 0 (else unused)
  const __nv_bfloat16* K;
  const float* qbar;
  int diag;
  // compact form (packed != 0): w holds, per row, the weights of the routed
  // chunks in increasing chunk order (entry k = the k-th set bit of the
  // row's mask); index (nullable) their chunk numbers, count (nullable) how
  // many there are
  int packed;
  int32_t* count;
  int32_t* index;
  int n_q, n_kv, seq, chunk, n_c, nw, kbar_rows, n_tiles, n_bg, pos_base;
  float xscale, e;
};

// named barrier over the 256 entmax threads (warps 0-7); returns the OR of p
__device__ __forceinline__ bool rows_sync_or(bool p) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred a, b;\n\t"
      "setp.ne.u32 a, %1, 0;\n\t"
      "bar.red.or.pred b, 1, 256, a;\n\t"
      "selp.u32 %0, 1, 0, b;\n\t}"
      : "=r"(r) : "r"((uint32_t)p) : "memory");
  return r != 0;
}
__device__ __forceinline__ void rows_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

template <bool SPLIT, int KIND>
__global__ void __launch_bounds__(288, 1) route_tc_kernel(
    const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmKb,
    const RouteTcParams prm) {
  constexpr int NPOS = SPLIT ? 4 : 8;           // positions per CTA
  constexpr int QROWS = NPOS * 16;              // rows of Q per CTA
  constexpr int QBOX = 128 * 128;               // 128 rows x 128 B (64 bf16 columns)
  constexpr int NQB = SPLIT ? 4 : 2;            // 64-column boxes of A (K = 256 or 128)
  constexpr int Q_BYTES = NQB * QBOX;
  constexpr int KT_ROWS = 256;                  // chunks per Kbar tile
  constexpr int KT_BOX = KT_ROWS * 128;
  constexpr int KT_BYTES = 2 * KT_BOX;          // one tile, d = 128
  extern __shared__ uint8_t smem_raw[];
  // 1024-byte aligned by pointer arithmetic on the shared array, so that the
  // compiler keeps the shared address space (and emits shared loads)
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint8_t* sQ = smem;
  uint8_t* sKt = smem + Q_BYTES;                // 2 tile slots
  // compact form: once the logits are in TMEM the Kbar tiles are free and
  // hold the rows' weights and mask words until they are compacted
  constexpr int NCMAX = SPLIT ? 1024 : 512;
  float* wst = reinterpret_cast<float*>(sKt);                          // [NPOS][NCMAX]
  uint32_t* mst = reinterpret_cast<uint32_t*>(sKt + NPOS * NCMAX * 4); // [NPOS][32]

  __shared__ __align__(8) uint64_t bar_q, bar_full[2], bar_empty[2], bar_logits;
  __shared__ uint32_t tmem_slot;
  __shared__ volatile int abort_s;
  __shared__ float xch[2][2][3][128];           // [parity][column half][value][row]: partial sums
  __shared__ float khat[NPOS][128];             // estimate_diagonal: the positions' diagonal summaries

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int tile = prm.n_tiles - 1 - (int)(blockIdx.x / prm.n_bg);    // late (heavy) tiles first
  const int bg = blockIdx.x % prm.n_bg;
  const int b = bg / prm.n_kv, g = bg % prm.n_kv;
  const int pos0 = prm.pos_base + tile * NPOS;
  const int c_i = pos0 / prm.chunk;
  const int n_elig = min(c_i, prm.n_c);
  // Kbar tiles: plain -- chunks [256 kt, 256 kt + 256); SPLIT -- tile pairs
  // (kt: chunks [256 kt, ...) for rows 0-63, [512 + 256 kt, ...) for rows 64-127)
  const int n_kt = SPLIT ? 2 : (n_elig + KT_ROWS - 1) / KT_ROWS;

  if (warp == 8) {
    tmem_alloc(&tmem_slot, 512);
    tmem_relinquish();
  }
  if (tid == 0) {
    mbar_init(&bar_q, 1);
    mbar_init(&bar_full[0], 1);
    mbar_init(&bar_full[1], 1);
    mbar_init(&bar_empty[0], 1);
    mbar_init(&bar_empty[1], 1);
    mbar_init(&bar_logits, 1);
    abort_s = 0;
    fence_mbar_init();
  }
  if (SPLIT) {
    // zero blocks of A_ext = [[Q, 0], [0, Q]]: rows 64-127 of K-boxes 0, 1 and
    // rows 0-63 of K-boxes 2, 3 (8 KB each; zeros are swizzle-invariant)
    for (int i = tid; i < 4 * 8192 / 16; i += blockDim.x) {
      const int blk = i / 512, off = (i % 512) * 16;
      const int base = blk * QBOX + (blk < 2 ? 8192 : 0);
      *reinterpret_cast<uint4*>(sQ + base + off) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;

  if (warp == 8) {
    // ---------------------------------------------------- TMA + MMA (one warp)
    constexpr uint32_t idL = idesc_bf16_f32(128, KT_ROWS, 0, 0);
    const bool leader = elect_one();
    if (n_kt > 0) {
      const int kbrow = bg * prm.kbar_rows;
      const int tile_bytes = SPLIT ? 2 * KT_BYTES : KT_BYTES;
      auto load_tile = [&](int kt, int slot) {
        if (SPLIT) {
          mbar_arrive_expect_tx(&bar_full[slot], 2 * KT_BYTES);
          for (int kb = 0; kb < 2; ++kb) {
            tma_load_2d(sKt + kb * KT_BOX, &tmKb, &bar_full[slot], kb * 64, kbrow + kt * KT_ROWS);
            tma_load_2d(sKt + KT_BYTES + kb * KT_BOX, &tmKb, &bar_full[slot], kb * 64,
                        kbrow + 512 + kt * KT_ROWS);
          }
        } else {
          mbar_arrive_expect_tx(&bar_full[slot], KT_BYTES);
          for (int kb = 0; kb < 2; ++kb)
            tma_load_2d(sKt + slot * KT_BYTES + kb * KT_BOX, &tmKb, &bar_full[slot], kb * 64,
                        kbrow + kt * KT_ROWS);
        }
      };
      if (leader) {
        tma_prefetch_desc(&tmQ);
        if (SPLIT) {
          mbar_arrive_expect_tx(&bar_q, 2 * 2 * QROWS * 128);
          for (int kb = 0; kb < 2; ++kb) {
            tma_load_3d(sQ + kb * QBOX, &tmQ, &bar_q, kb * 64, b * prm.n_q + g * 16, pos0);
            tma_load_3d(sQ + (2 + kb) * QBOX + 8192, &tmQ, &bar_q, kb * 64, b * prm.n_q + g * 16, pos0);
          }
          load_tile(0, 0);                   // one slot pair: tiles run one at a time
        } else {
          mbar_arrive_expect_tx(&bar_q, 2 * QBOX);
          for (int kb = 0; kb < 2; ++kb)
            tma_load_3d(sQ + kb * QBOX, &tmQ, &bar_q, kb * 64, b * prm.n_q + g * 16, pos0);
          for (int kt = 0; kt < 2 && kt < n_kt; ++kt) load_tile(kt, kt);
        }
      }
      __syncwarp();
      (void)tile_bytes;
      const uint64_t dQ0 = sw128_desc(smem_u32(sQ), 16, 1024);
      const uint64_t dK0 = sw128_desc(smem_u32(sKt), 16, 1024);
      bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_q, 0, &abort_s));
      for (int kt = 0; ok && kt < n_kt; ++kt) {
        const int slot = SPLIT ? 0 : (kt & 1);
        const uint32_t par = SPLIT ? (kt & 1) : ((kt >> 1) & 1);
        if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bar_full[slot], par, &abort_s)))) break;
        tc_fence_after();
        const uint32_t dst = tmem + kt * KT_ROWS;
        if (leader) {
#pragma unroll
          for (int kk = 0; kk < (SPLIT ? 16 : 8); ++kk) {
            // A: K-step kk of A_ext; B: low tile for kk < 8, high tile after
            const uint32_t offq = (kk >> 2) * QBOX + (kk & 3) * 32;
            const uint32_t offk = (SPLIT ? (kk >> 3) * KT_BYTES : slot * KT_BYTES) +
                                  ((kk >> 2) & 1) * KT_BOX + (kk & 3) * 32;
            tc_mma_ss(dst, dQ0 + (offq >> 4), dK0 + (offk >> 4), idL, kk > 0 ? 1u : 0u);
          }
          tc_commit(&bar_empty[slot]);
        }
        __syncwarp();
        const int nxt = SPLIT ? kt + 1 : kt + 2;
        if (nxt < n_kt) {
          // reload this slot once its MMAs have read it
          if (!(ok = __all_sync(0xffffffffu, mbar_wait(&bar_empty[slot], par, &abort_s)))) break;
          if (leader) load_tile(nxt, slot);
          __syncwarp();
        }
      }
      if (leader) tc_commit(&bar_logits);
      __syncwarp();
    }
  } else {
    // ---------------------------------------------------- entmax, two threads per row
    // warps w and w + 4 read the same TMEM lanes (rows); each takes half of
    // the row's 32-chunk blocks, and per-row totals are merged through
    // shared memory
    const int m = (warp & 3) * 32 + lane;                // TMEM lane = row of the MMA
    const int ch = warp >> 2;                            // column half of this thread
    const int half = SPLIT ? (m >> 6) : 0;               // SPLIT: chunk half of this row
    const int pl = SPLIT ? ((m & 63) >> 4) : (m >> 4);   // position within the CTA
    const int pos = pos0 + pl;
    const uint32_t trow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const int c_base = half * 512;                       // first chunk of this thread's range
    // estimate_diagonal: the query's own chunk c_i is one more candidate,
    // held in TMEM column c_i (right after the eligible ones; column
    // c_i - 512 of the upper half with SPLIT), so every pass below includes it
    const bool dg = prm.diag != 0 && n_elig > 0;
    const int cols = SPLIT ? (half ? n_elig - 512 + (dg ? 1 : 0) : 512) : n_elig + (dg ? 1 : 0);
    const int nblk = (cols + 31) >> 5;                   // the row's blocks (warp-uniform)
    const int nb0 = (nblk + 1) >> 1;
    const int bk_lo = ch ? nb0 : 0, bk_hi = ch ? nblk : nb0;   // this thread's blocks
    const size_t rowidx = (size_t)bg * prm.seq + pos;
    float* wrow = prm.w + rowidx * prm.n_c;
    uint32_t* mrow = prm.mask + rowidx * prm.nw;
    const float xs = prm.xscale, e = prm.e;
    const int c_end = n_elig;
    // row totals of up to three values over the threads that share the row
    // (the two column halves; with SPLIT also the lanes m and m ^ 64 of the
    // two chunk halves), summed (op 1) or maxed (op 0) in one fixed order so
    // that every thread of the row holds the same result; all 256 threads
    // call it (double-buffered, one barrier per call)
    int xpar = 0;
    auto merge = [&](float& a, float& bb, float& cc, int op) {
      xch[xpar][ch][0][m] = a;
      xch[xpar][ch][1][m] = bb;
      xch[xpar][ch][2][m] = cc;
      rows_sync();
      float v[3];
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const int m0 = SPLIT ? (m & 63) : m;
        float t0 = xch[xpar][0][k][m0], t1 = xch[xpar][1][k][m0];
        float r = op == 0 ? fmaxf(t0, t1) : t0 + t1;
        if (SPLIT) {
          const float u0 = xch[xpar][0][k][m0 + 64], u1 = xch[xpar][1][k][m0 + 64];
          r = op == 0 ? fmaxf(r, fmaxf(u0, u1)) : r + (u0 + u1);
        }
        v[k] = r;
      }
      a = v[0];
      if (op != 0) { bb = v[1]; cc = v[2]; }
      xpar ^= 1;
    };
    int blocks_written = 0;                              // 32-chunk blocks of w written
    // estimate_diagonal: stage 0's summary of the keys each position may see
    // in its own chunk (warp p, position p), then this row's scaled logit
    // against it; computed while the logit MMAs run
    float xd = -INFINITY;
    if (dg) {
      if (warp < NPOS)
        summarize_chunk_warp<__nv_bfloat16, 128, 4, float>(
            prm.K + ((size_t)bg * prm.seq + (size_t)c_i * prm.chunk) * 128, prm.qbar + g * 128,
            khat[warp], pos0 + warp - c_i * prm.chunk + 1, lane);
      rows_sync();
      if (mbar_wait(&bar_q, 0, &abort_s)) {
        // Q row (m & 63 with SPLIT: rows 64-127 repeat rows 0-63) from the
        // 128-byte-swizzled tile, boxes 0 and 1 (columns 0-63, 64-127)
        const int qr = SPLIT ? (m & 63) : m;
        float acc = 0.f;
#pragma unroll
        for (int kb = 0; kb < 2; ++kb) {
          const uint8_t* qrow = sQ + kb * QBOX + (qr >> 3) * 1024 + (qr & 7) * 128;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const uint4 v = *reinterpret_cast<const uint4*>(qrow + ((cc ^ (qr & 7)) << 4));
            const __nv_bfloat16* qv = reinterpret_cast<const __nv_bfloat16*>(&v);
            const float* kh = khat[pl] + kb * 64 + cc * 8;
#pragma unroll
            for (int e2 = 0; e2 < 8; ++e2) acc = fmaf(__bfloat162float(qv[e2]), kh[e2], acc);
          }
        }
        xd = acc * prm.xscale;
      }
    }
    bool have = n_kt > 0 && mbar_wait(&bar_logits, 0, &abort_s);
    have = !rows_sync_or(!have);                         // all 256 threads agree
    if (have) {
      tc_fence_after();
      float dummy1 = 0.f, dummy2 = 0.f;
      // pass 0: x = (alpha - 1) gamma z written back over z, -inf past the
      // eligible chunks (later passes need no bounds checks), and the row max
      float mx = -INFINITY;
      {
        const uint64_t xs2 = f2_pack(xs, xs);
        for (int bk = bk_lo; bk < bk_hi; ++bk) {
          float x[32];
          tmem_ld32(trow + bk * 32, x);
          const int cb = c_base + bk * 32;
#pragma unroll
          for (int i = 0; i < 32; i += 2) f2_unpack(f2_mul(f2_pack(x[i], x[i + 1]), xs2), x[i], x[i + 1]);
          if (cb + 32 > c_end) {                         // warp-uniform: the last blocks only
#pragma unroll
            for (int i = 0; i < 32; ++i) x[i] = cb + i < c_end ? x[i] : (cb + i == c_i ? xd : -INFINITY);
          }
#pragma unroll
          for (int i = 0; i < 32; i += 2) mx = fmax3(mx, x[i], x[i + 1]);
          tmem_st32(trow + bk * 32, x);
        }
        tmem_wait_st();
      }
      merge(mx, dummy1, dummy2, 0);
      // sums over the row at threshold t: S0 = sum d^e and S1 = sum d^(e-1)
      // (times e; the count for sparsemax), d = [x - t]_+; with want_k also
      // the support size K = #(x > t).  Pairs of values per f32x2 op.
      auto row_sums = [&](float t, bool want_k, float& S0, float& S1, float& K) {
        const uint64_t nt2 = f2_pack(-t, -t);
        uint64_t a0 = 0ull, a1 = 0ull, b0 = 0ull, b1 = 0ull;   // packed (+0, +0)
        float k0 = 0.f, g0 = 0.f, g1 = 0.f;
        for (int bk = bk_lo; bk < bk_hi; ++bk) {
          float x[32];
          tmem_ld32(trow + bk * 32, x);
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float d0, d1;
            f2_unpack(f2_add(f2_pack(x[i], x[i + 1]), nt2), d0, d1);
            const float r0 = fmaxf(d0, 0.f), r1 = fmaxf(d1, 0.f);
            if (want_k) k0 += (d0 > 0.f ? 1.f : 0.f) + (d1 > 0.f ? 1.f : 0.f);
            const uint64_t rr = f2_pack(r0, r1);
            if (KIND == kEntmax15) {
              if (i & 2) { a1 = f2_fma(rr, rr, a1); b1 = f2_add(b1, rr); }
              else { a0 = f2_fma(rr, rr, a0); b0 = f2_add(b0, rr); }
            } else if (KIND == kSparsemax) {
              if (i & 2) a1 = f2_add(a1, rr);
              else a0 = f2_add(a0, rr);
              if (!want_k) g0 += (d0 > 0.f ? 1.f : 0.f) + (d1 > 0.f ? 1.f : 0.f);
            } else {
              const float p0 = entmax_pow<KIND>(r0, e), p1 = entmax_pow<KIND>(r1, e);
              g0 += p0 + p1;
              g1 += (r0 > 0.f ? p0 / r0 : 0.f) + (r1 > 0.f ? p1 / r1 : 0.f);
            }
          }
        }
        float u0, u1, u2, u3;
        f2_unpack(f2_add(a0, a1), u0, u1);
        f2_unpack(f2_add(b0, b1), u2, u3);
        if (KIND == kEntmax15) { S0 = u0 + u1; S1 = u2 + u3; }
        else if (KIND == kSparsemax) { S0 = u0 + u1; S1 = want_k ? k0 : g0; }
        else { S0 = g0; S1 = g1; }
        K = k0;
      };
      // Newton on the e-norm from tau = max - 1
      float tau = mx - 1.f;
      bool conv = false;
      for (int it = 0; it < 48; ++it) {
        float s0, s1, s2;
        row_sums(tau, false, s0, s1, s2);
        s2 = 0.f;
        merge(s0, s1, s2, 1);
        if (!conv) {
          const float f = s0 - 1.f;
          if (!(f > 0.f) || !(s1 > 0.f)) {
            conv = true;
          } else {
            float step;
            if (KIND == kEntmax15) step = (s0 - sqrtf(s0)) / s1;
            else if (KIND == kSparsemax) step = f / s1;
            else { const float nrm = ex2f(lg2f(s0) / e); step = (nrm - 1.f) * s0 / (nrm * s1); }
            const float nt = tau + step;
            if (!(nt > tau)) conv = true;
            else tau = nt;
            if (f < 1e-6f) conv = true;
          }
        }
        const bool more = rows_sync_or(!conv);         // uniform over the CTA
        if (!more) break;
      }
      // alpha = 1.5 / 2: the exact root on the support S = {x > tau} found
      float tc = tau, kk = 0.f;
      bool cand = false;
      if (KIND != kEntmaxGeneric) {
        float d2, d1;
        row_sums(tau, true, d2, d1, kk);                 // entmax15: sum d^2, sum d
        if (KIND == kSparsemax) d1 = d2;                 // sparsemax: sum d
        merge(d1, d2, kk, 1);
        if (KIND == kEntmax15) {
          const float disc = d1 * d1 - kk * (d2 - 1.f);
          if (kk > 0.f && disc >= 0.f) { tc = tau + (d2 - 1.f) / (d1 + sqrtf(disc)); cand = true; }
        } else if (kk > 0.f) {
          tc = tau + (d1 - 1.f) / kk;
          cand = true;
        }
      }
      // p at t, GQA mean over the 16 lanes of this position, w and mask.
      // With `count` it also returns #(x > t): the candidate root is kept
      // only if that equals #(x > tau), i.e. no element lies in (tau, tc].
      const int h = lane & 15;
      const float invG = 1.f / 16.f;
      auto write_pass = [&](float t, bool count) -> float {
        const uint64_t nt2 = f2_pack(-t, -t);
        float cnt = 0.f;
        for (int bk = bk_lo; bk < bk_hi; ++bk) {
          float x[32];
          tmem_ld32(trow + bk * 32, x);
          const int c0 = c_base + bk * 32;
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float d0, d1;
            f2_unpack(f2_add(f2_pack(x[i], x[i + 1]), nt2), d0, d1);
            if (count) cnt += (d0 > 0.f ? 1.f : 0.f) + (d1 > 0.f ? 1.f : 0.f);
            v[i] = entmax_pow<KIND>(fmaxf(d0, 0.f), e);
            v[i + 1] = entmax_pow<KIND>(fmaxf(d1, 0.f), e);
          }
          // reduce-scatter over the 16 heads: lane h ends with chunks c0+2h, c0+2h+1
#pragma unroll
          for (int sh = 8, len = 16; sh >= 1; sh >>= 1, len >>= 1) {
            const bool up = (h & sh) != 0;
#pragma unroll
            for (int i = 0; i < len; ++i) {
              const float send = up ? v[i] : v[len + i];
              const float keep = up ? v[len + i] : v[i];
              v[i] = keep + __shfl_xor_sync(0xffffffffu, send, sh);
            }
          }
          const int c = c0 + 2 * h;
          const float w0 = v[0] * invG, w1 = v[1] * invG;
          if (c0 < prm.n_c) {
            // the query's own chunk (estimate_diagonal) is never a mask bit
            uint32_t bits = ((w0 > 0.f && c != c_i ? 1u : 0u) | (w1 > 0.f && c + 1 != c_i ? 2u : 0u))
                            << (2 * h);
#pragma unroll
            for (int sh = 1; sh < 16; sh <<= 1) bits |= __shfl_xor_sync(0xffffffffu, bits, sh);
            if (prm.packed) {
              // staged in shared memory; compacted once the row is complete
              wst[pl * NCMAX + c] = w0;
              wst[pl * NCMAX + c + 1] = w1;
              if (h == 0) mst[pl * 32 + (c0 >> 5)] = bits;
            } else {
              // two scalar stores: with an odd n_c the row start is only
              // 4-byte aligned (the half-warp still writes one contiguous
              // 128-byte span)
              if (c < prm.n_c) wrow[c] = w0;
              if (c + 1 < prm.n_c) wrow[c + 1] = w1;
              if (h == 0) mrow[c0 >> 5] = bits;
            }
          }
        }
        return cnt;
      };
      float kt = write_pass(cand ? tc : tau, cand);
      if (KIND != kEntmaxGeneric) {
        // a candidate that dropped an element of S: redo those rows at tau
        // (rare; the whole warp redoes, as its positions' sums are shared)
        float none = 0.f;
        merge(kt, none, dummy2, 1);
        const bool bad = cand && kt != kk;
        const bool redo = rows_sync_or(bad);
        if (redo) write_pass(bad || !cand ? tau : tc, false);
      }
      blocks_written = nblk;
      if (prm.packed) {
        // compact form: warp p writes position p's routed chunks in order
        // (rank = set bits before them), its mask words and count
        rows_sync();
        if (warp < NPOS) {
          const size_t rix = (size_t)bg * prm.seq + pos0 + warp;
          float* wq = prm.w + rix * prm.n_c;
          int32_t* iq = prm.index ? prm.index + rix * prm.n_c : nullptr;
          uint32_t* mq = prm.mask + rix * prm.nw;
          const int nwr = (n_elig + 31) >> 5;            // words holding routed chunks
          int base = 0;
          for (int k = 0; k < prm.nw; ++k) {
            uint32_t bits = k < nwr ? mst[warp * 32 + k] : 0u;
            if (k * 32 + 32 > n_elig) bits &= n_elig > k * 32 ? (1u << (n_elig - k * 32)) - 1u : 0u;
            if ((bits >> lane) & 1u) {
              const int at = base + __popc(bits & ((1u << lane) - 1u));
              wq[at] = wst[warp * NCMAX + k * 32 + lane];
              if (iq) iq[at] = k * 32 + lane;
            }
            if (lane == 0) mq[k] = bits;
            base += __popc(bits);
          }
          if (lane == 0 && prm.count) prm.count[rix] = base;
        }
      }
    }
    // mask words / w columns not written above are 0: words
    // [c_base / 32 + blocks_written, nw) of this position's row (for SPLIT the
    // lower half covers all of words 0-15 whenever it has work)
    const int zfirst = prm.packed ? (have ? prm.nw : 0) : (c_base >> 5) + blocks_written;
    const int zlast = SPLIT && !half ? min(16, prm.nw) : prm.nw;
    if (prm.packed && !have && ch == 0 && (!SPLIT || !half) && (lane & 15) == 0 && prm.count)
      prm.count[rowidx] = 0;                             // no eligible chunk: an empty row
    for (int k = zfirst + (lane & 15); ch == 0 && k < zlast; k += 16) {
      mrow[k] = 0u;
      if (prm.packed) continue;
      for (int i = 0; i < 32 && k * 32 + i < prm.n_c; ++i) wrow[k * 32 + i] = 0.f;
      // estimate_diagonal on a row of the first chunk: the diagonal is the
      // only candidate, weight 1
      if (k == 0 && prm.diag && n_elig == 0) wrow[c_i] = 1.f;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 8) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

inline size_t route_tc_smem_bytes(bool split) {
  // A (2 or 4 boxes of 16 KB) + two Kbar tiles of 64 KB + alignment slack
  return (size_t)(split ? 4 : 2) * 128 * 128 + (size_t)2 * 2 * 256 * 128 + 1024;
}

template <bool SPLIT, int KIND>
cudaError_t launch_route_tc_k(const CUtensorMap& tq, const CUtensorMap& tk, const RouteTcParams& prm,
                              cudaStream_t st) {
  auto kern = route_tc_kernel<SPLIT, KIND>;
  size_t smem = route_tc_smem_bytes(SPLIT);
  // the CTA holds all 512 TMEM columns: keep it alone on its SM
  if (smem < 118 * 1024) smem = 118 * 1024;
  cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (err != cudaSuccess) return err;
  kern<<<(unsigned)(prm.n_tiles * prm.n_bg), 288, smem, st>>>(tq, tk, prm);
  return cudaGetLastError();
}

// Q [b, n_q, seq, 128] and Kbar [b, n_kv, seq / chunk, 128] bf16; G = 16,
// n_c <= 1024.  Positions with at most 512 eligible chunks run 8 per CTA;
// the rest (n_c > 512 only) run 4 per CTA through the split variant.
template <bool SPLIT>
cudaError_t launch_route_tc_part(const __nv_bfloat16* Q, const CUtensorMap& tk, RouteTcParams prm,
                                 int batch, int pos_begin, int pos_end, float alpha,
                                 cudaStream_t st) {
  const int npos = SPLIT ? 4 : 8;
  if (pos_end <= pos_begin) return cudaSuccess;
  CUtensorMap tq;
  const uint64_t dims[3] = {128, (uint64_t)batch * prm.n_q, (uint64_t)prm.seq};
  const uint64_t str[2] = {(uint64_t)prm.seq * 128 * 2, 128 * 2};
  const uint32_t box[3] = {64, 16, (uint32_t)npos};
  if (!make_tmap(&tq, Q, 3, dims, str, box)) return cudaErrorInvalidValue;
  prm.pos_base = pos_begin;
  prm.n_tiles = (pos_end - pos_begin) / npos;
  if (alpha == 1.5f) return launch_route_tc_k<SPLIT, kEntmax15>(tq, tk, prm, st);
  if (alpha == 2.f) return launch_route_tc_k<SPLIT, kSparsemax>(tq, tk, prm, st);
  return launch_route_tc_k<SPLIT, kEntmaxGeneric>(tq, tk, prm, st);
}

// K, qbar: non-null for estimate_diagonal, else both null.  packed: w is the
// compact form (count, index nullable), else dense.
inline cudaError_t launch_route_tc(const __nv_bfloat16* Q, const __nv_bfloat16* Kbar, float* w,
                                   uint32_t* mask, const __nv_bfloat16* K, const float* qbar,
                                   int batch, int n_q, int n_kv, int seq, int chunk, float alpha,
                                   float gamma, cudaStream_t st, bool packed = false,
                                   int32_t* count = nullptr, int32_t* index = nullptr) {
  const int n_c = (seq + chunk - 1) / chunk;
  CUtensorMap tk;
  {
    const uint64_t dims[2] = {128, (uint64_t)batch * n_kv * (seq / chunk)};
    const uint64_t str[1] = {128 * 2};
    const uint32_t box[2] = {64, 256};
    if (!make_tmap(&tk, Kbar, 2, dims, str, box)) return cudaErrorInvalidValue;
  }
  RouteTcParams prm;
  prm.w = w;
  prm.mask = mask;
  prm.K = K;
  prm.qbar = qbar;
  prm.diag = K != nullptr;
  prm.packed = packed ? 1 : 0;
  prm.count = count;
  prm.index = index;
  prm.n_q = n_q;
  prm.n_kv = n_kv;
  prm.seq = seq;
  prm.chunk = chunk;
  prm.n_c = n_c;
  prm.nw = (n_c + 31) / 32;
  prm.kbar_rows = seq / chunk;
  prm.n_bg = batch * n_kv;
  prm.xscale = (alpha - 1.f) * gamma;
  prm.e = 1.f / (alpha - 1.f);
  const int split_from = min(seq, 512 * chunk);     // first position with c_i >= 512
  cudaError_t err = launch_route_tc_part<false>(Q, tk, prm, batch, 0, split_from, alpha, st);
  if (err != cudaSuccess) return err;
  return launch_route_tc_part<true>(Q, tk, prm, batch, split_from, seq, alpha, st);
}

}  // namespace dash
