// Bidirectional local-window attention on tcgen05 tensor cores (prefill, bf16, d = 128):
// the sliding window of the non-route layers (MODE 0: o bf16 and lse) and the route layer's
// local window (MODE 1: normalised o_loc fp32 and lambda_loc, read by the chunk kernel).
// Definition as in window_attn.cuh: W(p) = { j : |p - j| <= w, 0 <= j < L } (Prefilling-dLLM
// v2, abstract and Table 3), every slot included.
//
//   CTA = 16 consecutive query tokens x one KV group.  The 128 rows of the tile are
//   (token, head slot) pairs, token-major, 8 head slots per token (slots past the group's
//   heads are computed and dropped).  The keys the tile's windows cover are streamed in
//   tiles of 128 keys by TMA, twice:
//     pass 1   S = Q K^T  (tcgen05.mma M = 128, N = 128, K = 128 -> tensor memory); the
//              softmax warps read S and keep each row's maximum over its window;
//     pass 2   S again, P = 2^(S - max) in bf16 written to shared memory (row sums kept in
//              fp32), O += P V (M = 128, N = 128 head dims, K = 128 keys) in tensor memory.
//   Knowing the maximum before any P is formed means O is never rescaled: the price is the
//   second S, cheaper on these tensor cores than reading and rewriting O between tiles.
//
// Warp roles (384 threads): warp 0 issues the MMAs (warp-collective, one elected lane),
// warp 1 issues the TMA loads (one lane), warps 4-11 own the 128 rows for the softmax and
// the epilogue: TMEM lane quarter = warp % 4, one row per thread, warps 4-7 the first 64
// keys of each tile (and head dims 0-63), warps 8-11 the other 64; the two halves of a
// row combine their maximum (end of pass 1) and sum (end of pass 2) through shared memory.
// Tensor memory: S in two buffers of 128 columns (the MMAs of tile t + 1 overlap the
// softmax of tile t), O in 128 columns.
// Shared memory (from a 1024-byte-aligned base): Q 32 KB (token-major, 2 KB per token: head
// rows for columns 0-63, then 64-127), two K/V stages of 64 KB (K then V, each
// [2 column halves][128 keys][128 B]), P 32 KB ([2 key halves][128 rows][128 B]); all
// 128-byte swizzled.
// Every wait is bounded; after a timeout the kernel records RDL_ERR_TIMEOUT, every role
// stops, the MMAs in flight drain, the last TMA loads land, tensor memory is freed.
#pragma once
#include "common.cuh"
#include "tc.cuh"

namespace rdl {

constexpr int WT_TOK = 16;                     // query tokens per CTA (x 8 head slots = M)
constexpr int WT_KEYS = 128;                   // keys per tile
constexpr int WT_THREADS = 384;
constexpr int WT_OFF_Q = 0;
constexpr int WT_OFF_KV = 32768;               // stage s: K at + 65536 s, V at + 32768
constexpr int WT_OFF_P = WT_OFF_KV + 2 * 65536;
constexpr int WT_OFF_BAR = WT_OFF_P + 32768;
constexpr int WT_OFF_RED = WT_OFF_BAR + 256;      // [2 halves][128 rows] fp32 row reductions
constexpr int WT_SMEM = WT_OFF_RED + 1024 + 1024;   // + alignment slack
constexpr uint32_t WT_TCOLS = 512;             // S0 [0,128), S1 [128,256), O [256,384)
static_assert(WT_SMEM <= 227 * 1024, "shared memory");

template <int MODE>
__global__ void __launch_bounds__(WT_THREADS, 1)
    window_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap kmap,
                     const __grid_constant__ CUtensorMap vmap, const int32_t* __restrict__ q_pos, int L, int Lq,
                     int Hq, int Hkv, int w, __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                     float* __restrict__ o_loc, float* __restrict__ lam_loc) {
  constexpr int D = 128;
  extern __shared__ unsigned char wt_raw[];
  unsigned char* sm = wt_raw + ((1024u - (smem_u32(wt_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + WT_OFF_BAR);
  uint64_t* qfull = bars;          // Q landed
  uint64_t* full = bars + 1;       // [2] K (pass 1) or K and V (pass 2) of a stage landed
  uint64_t* empty = bars + 3;      // [2] stage consumed (commit)
  uint64_t* sfull = bars + 5;      // [2] S buffer written (commit)
  uint64_t* sempty = bars + 7;     // [2] S buffer read (8 softmax warps)
  uint64_t* pfull = bars + 9;      // P written (8 softmax warps)
  uint64_t* pempty = bars + 10;    // P consumed by the PV MMAs (commit)
  uint64_t* ofull = bars + 11;     // every PV MMA complete (commit)
  uint64_t* mdone = bars + 12;     // every MMA of the issuer complete
  uint64_t* redbar = bars + 13;    // [2] row maxima / row sums of both halves stored (8 warps)
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 15);
  int* abort_f = reinterpret_cast<int*>(tslot + 1);
  int* pos_s = abort_f + 1;        // [WT_TOK]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = Hq / Hkv;
  const int i0 = blockIdx.x * WT_TOK;
  const int bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv;

  if (tid == 0) {
    tc::mbar_init(qfull, 1);
    for (int j = 0; j < 2; ++j) {
      tc::mbar_init(&full[j], 1);
      tc::mbar_init(&empty[j], 1);
      tc::mbar_init(&sfull[j], 1);
      tc::mbar_init(&sempty[j], 8);
    }
    tc::mbar_init(pfull, 8);
    tc::mbar_init(pempty, 1);
    tc::mbar_init(ofull, 1);
    tc::mbar_init(mdone, 1);
    tc::mbar_init(&redbar[0], 8);
    tc::mbar_init(&redbar[1], 8);
    *abort_f = 0;
    tc::mbar_fence_init();
  }
  if (tid < WT_TOK) {
    const int i = i0 + tid;
    pos_s[tid] = i < Lq ? (q_pos ? q_pos[(size_t)b * Lq + i] : i) : INT_MIN;
  }
  if (warp == 0) {
    tc::tmem_alloc(tslot, WT_TCOLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tslot;
  // keys the tile's windows cover: [kbeg, kend), in tiles of 128
  int pmin = INT_MAX, pmax = INT_MIN;
#pragma unroll
  for (int t = 0; t < WT_TOK; ++t)
    if (pos_s[t] != INT_MIN) {
      pmin = min(pmin, pos_s[t]);
      pmax = max(pmax, pos_s[t]);
    }
  const int kbeg = pmax >= pmin ? max(0, pmin - w) : 0;
  const int kend = pmax >= pmin ? min(L, pmax + w + 1) : 0;
  const int nt = kend > kbeg ? (kend - kbeg + WT_KEYS - 1) / WT_KEYS : 0;
  const int krow0 = (b * Hkv + g) * L + kbeg;

  if (warp == 1) {
    // ---------------- TMA producer
    if (lane == 0 && nt > 0) {
      tc::mbar_arrive_expect_tx(qfull, 32768u);
      tc::tma_load_4d(sm + WT_OFF_Q, &qmap, 0, g * G, 0, b * Lq + i0, qfull);
      int u = 0;
      for (int pass = 0; pass < 2; ++pass)
        for (int t = 0; t < nt; ++t, ++u) {
          const int st = u & 1, n = u >> 1;
          if ((n > 0 && !tc::mbar_wait(&empty[st], (unsigned)(n - 1) & 1u)) || *(volatile int*)abort_f) {
            *(volatile int*)abort_f = 1;
            break;
          }
          unsigned char* kst = sm + WT_OFF_KV + st * 65536;
          tc::mbar_arrive_expect_tx(&full[st], pass ? 65536u : 32768u);
          tc::tma_load_3d(kst, &kmap, 0, krow0 + WT_KEYS * t, 0, &full[st]);
          if (pass) tc::tma_load_3d(kst + 32768, &vmap, 0, krow0 + WT_KEYS * t, 0, &full[st]);
        }
      // the last load issued into each stage has landed before the CTA may exit
      for (int x = max(0, u - 2); x < u; ++x) (void)tc::mbar_wait(&full[x & 1], (unsigned)(x >> 1) & 1u);
      (void)tc::mbar_wait(qfull, 0);
    }
    __syncwarp();
  } else if (warp == 0) {
    // ---------------- MMA issuer (warp-collective)
    const uint32_t idesc_s = tc::idesc_bf16(128, 128, false, false);
    const uint32_t idesc_pv = tc::idesc_bf16(128, 128, false, true);
    const uint64_t dQ = tc::sdesc(smem_u32(sm + WT_OFF_Q), 16, 2048);
    const uint64_t dP = tc::sdesc(smem_u32(sm + WT_OFF_P), 16, 1024);
    bool issued = false, ok = nt > 0;
    int k = 0;                       // S buffers used so far
    auto wait_all = [&](uint64_t* bar, unsigned ph) -> bool {
      const bool r = tc::mbar_wait(bar, ph) && !*(volatile int*)abort_f;
      return __all_sync(0xffffffffu, r);
    };
    // S of the tile in stage st into buffer k & 1
    auto issue_s = [&](int st) -> bool {
      const int sb = k & 1;
      if (!wait_all(&sempty[sb], ((unsigned)(k >> 1) & 1u) ^ 1u)) return false;
      tc::tc_fence_after();
      const uint64_t dK = tc::sdesc(smem_u32(sm + WT_OFF_KV + st * 65536), 16, 1024);
      const uint32_t dS = tbase + (uint32_t)(sb * 128);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc::mma_bf16_ss_warp(dS, dQ + (uint64_t)((ks >> 2) * 64 + (ks & 3) * 2),
                             dK + (uint64_t)((ks >> 2) * 1024 + (ks & 3) * 2), idesc_s, ks > 0);
      tc::mma_commit_warp(&sfull[sb]);
      ++k;
      issued = true;
      return true;
    };
    if (ok) ok = wait_all(qfull, 0);
    int u = 0;
    for (int t = 0; t < nt && ok; ++t, ++u) {          // pass 1
      const int st = u & 1;
      if (!wait_all(&full[st], (unsigned)(u >> 1) & 1u) || !issue_s(st)) { ok = false; break; }
      tc::mma_commit_warp(&empty[st]);
    }
    const int u2 = u;                                  // pass 2: S of tile t + 1 before PV of t
    if (ok && nt > 0) ok = wait_all(&full[u2 & 1], (unsigned)(u2 >> 1) & 1u) && issue_s(u2 & 1);
    for (int t = 0; t < nt && ok; ++t) {
      const int ut = u2 + t, st = ut & 1;
      if (t + 1 < nt) {
        const int u1 = ut + 1;
        if (!wait_all(&full[u1 & 1], (unsigned)(u1 >> 1) & 1u) || !issue_s(u1 & 1)) { ok = false; break; }
      }
      if (!wait_all(pfull, (unsigned)t & 1u)) { ok = false; break; }
      tc::tc_fence_after();
      const uint64_t dV = tc::sdesc(smem_u32(sm + WT_OFF_KV + st * 65536 + 32768), 16384, 1024);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        tc::mma_bf16_ss_warp(tbase + 256u, dP + (uint64_t)((ks >> 2) * 1024 + (ks & 3) * 2),
                             dV + (uint64_t)(ks * 128), idesc_pv, (t | ks) != 0);
      tc::mma_commit_warp(pempty);
      tc::mma_commit_warp(&empty[st]);
    }
    if (ok && nt > 0) tc::mma_commit_warp(ofull);
    if (!ok && lane == 0) *(volatile int*)abort_f = 1;
    if (issued) tc::mma_commit_warp(mdone); else tc::mbar_arrive_warp(mdone);
    (void)tc::mbar_wait(mdone, 0);
    __syncwarp();
  } else if (warp >= 4 && warp < 12) {
    // ---------------- softmax and epilogue: row r = (token r / 8, head slot r % 8); this
    // thread's half of the row: keys 64 hf .. 64 hf + 63 of each tile, head dims likewise
    const int quad = warp & 3, hf = (warp - 4) >> 2, r = 32 * quad + lane, tok = r >> 3, hs = r & 7;
    const int p = pos_s[tok];
    const bool rowv = p != INT_MIN && hs < G;
    const int jlo = max(0, p - w), jhi = min(L - 1, p + w);       // the row's window
    const float sl2 = rsqrtf((float)D) * LOG2E;
    const uint32_t lrow = tc::taddr(tbase, 32 * quad, 0);
    float* red = reinterpret_cast<float*>(sm + WT_OFF_RED);        // [2][128]
    float m = -INFINITY, l = 0.f;
    bool ok = nt > 0;
    int k = 0;
    auto wait_all = [&](uint64_t* bar, unsigned ph) -> bool {
      const bool rr = tc::mbar_wait(bar, ph) && !*(volatile int*)abort_f;
      return __all_sync(0xffffffffu, rr);
    };
    // both halves of every row have stored their value (bounded: a half that gave up never
    // arrives, and its partner then gives up too)
    auto sync_halves = [&](int x) -> bool {
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&redbar[x]);
      return wait_all(&redbar[x], 0);
    };
    for (int pass = 0; pass < 2 && ok; ++pass) {
      if (pass == 1) {
        // the row maximum: the two halves' maxima through shared memory
        red[hf * 128 + r] = m;
        if (!sync_halves(0)) { ok = false; break; }
        m = fmaxf(red[r], red[128 + r]);
      }
      const float ms = m == -INFINITY ? 0.f : m;
      for (int t = 0; t < nt; ++t, ++k) {
        const int sb = k & 1;
        if (!wait_all(&sfull[sb], (unsigned)(k >> 1) & 1u)) { ok = false; break; }
        if (pass == 1 && !wait_all(pempty, ((unsigned)t & 1u) ^ 1u)) { ok = false; break; }
        tc::tc_fence_after();
        const int jt = kbeg + WT_KEYS * t;
#pragma unroll 1
        for (int c = 2 * hf; c < 2 * hf + 2; ++c) {
          float v[32];
          tc::tmem_ld32(lrow + (uint32_t)(sb * 128 + 32 * c), v);
          tc::tmem_wait_ld();
          const int j0 = jt + 32 * c;
          if (pass == 0) {
#pragma unroll
            for (int e = 0; e < 32; ++e) {
              const int j = j0 + e;
              if (rowv && j >= jlo && j <= jhi) m = fmaxf(m, v[e] * sl2);
            }
          } else {
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const int j = j0 + e;
              const float p0 = (rowv && j >= jlo && j <= jhi) ? fast_exp2(v[e] * sl2 - ms) : 0.f;
              const float p1 = (rowv && j + 1 >= jlo && j + 1 <= jhi) ? fast_exp2(v[e + 1] * sl2 - ms) : 0.f;
              l += p0 + p1;
              pk[e >> 1] = pack_bf16(p0, p1);
            }
            // keys 32c..32c+31 of the row: key half c / 2, 16-byte units 4 (c % 2) .. + 3
            unsigned char* prow = sm + WT_OFF_P + (c >> 1) * 16384 + r * 128;
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
              const int unit = (c & 1) * 4 + uu;
              *reinterpret_cast<uint4*>(prow + ((unit ^ (r & 7)) << 4)) =
                  make_uint4(pk[4 * uu], pk[4 * uu + 1], pk[4 * uu + 2], pk[4 * uu + 3]);
            }
          }
        }
        if (pass == 1) tc::fence_proxy_async();       // P is read by the tensor cores
        tc::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          tc::mbar_arrive(&sempty[sb]);
          if (pass == 1) tc::mbar_arrive(pfull);
        }
      }
    }
    // ---- epilogue: O / l for this half of the row, and the row's log-sum-exp
    bool eok = ok && wait_all(ofull, 0);
    if (eok) {
      red[hf * 128 + r] = l;            // pass 1's reads of red are behind the pass 2 barriers
      eok = sync_halves(1);
    }
    if (eok) {
      l = red[r] + red[128 + r];
      tc::tc_fence_after();
      const int i = i0 + tok, h = g * G + hs;
      const bool st_ok = rowv && i < Lq;
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const size_t rowoff = ((size_t)(b * Lq + (st_ok ? i : 0)) * Hq + h) * D;
#pragma unroll 1
      for (int c = 2 * hf; c < 2 * hf + 2; ++c) {
        float v[32];
        tc::tmem_ld32(lrow + (uint32_t)(256 + 32 * c), v);
        tc::tmem_wait_ld();
        if (!st_ok) continue;
        if (MODE == 0) {
          uint32_t pk[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) pk[e >> 1] = pack_bf16(v[e] * inv, v[e + 1] * inv);
          uint4* dst = reinterpret_cast<uint4*>(o + rowoff + 32 * c);
#pragma unroll
          for (int uu = 0; uu < 4; ++uu) dst[uu] = make_uint4(pk[4 * uu], pk[4 * uu + 1], pk[4 * uu + 2], pk[4 * uu + 3]);
        } else {
          float4* dst = reinterpret_cast<float4*>(o_loc + rowoff + 32 * c);
#pragma unroll
          for (int uu = 0; uu < 8; ++uu)
            dst[uu] = make_float4(v[4 * uu] * inv, v[4 * uu + 1] * inv, v[4 * uu + 2] * inv, v[4 * uu + 3] * inv);
        }
      }
      if (st_ok && hf == 0) {
        const float ls = l > 0.f ? (m + __log2f(l)) * LN2 : -INFINITY;
        float* lo = MODE == 0 ? lse : lam_loc;
        if (lo) lo[(size_t)(b * Hq + h) * Lq + i] = ls;
      }
    } else if (lane == 0) {
      *(volatile int*)abort_f = 1;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) tc::tmem_dealloc(tbase, WT_TCOLS);
}

}  // namespace rdl
