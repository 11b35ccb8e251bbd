// Route score for prefill on tcgen05 tensor cores (bf16 q, d = 128, residual rank 64).
// Same definition and split as score_mma.cuh (Prefilling-dLLM v2, Figure 3 caption):
//     z = tau * (q_h . s + t . s'_c,h) - lambda * H,   s'_c,h = W_up,h s_c,h,
// with s = s_hi + s_lo, s' = s'_hi + s'_lo and t = t_hi + t_lo split into bf16 terms and the
// five products q.s_hi + q.s_lo + t_hi.s'_hi + t_hi.s'_lo + t_lo.s'_hi in fp32.
//
//   CTA = (64 chunks, 128 query rows, batch x KV group); the group's heads in turn.  Per
//   head, by TMA: q_h [128 rows x 128] and the 64 chunks' split rows of sprep_kernel.  The
//   products are three MMA groups into tensor memory, the chunk operand stacked along N
//   so that one read of an A tile serves two split terms:
//     DA  = q_h . [s_hi ; s_lo]^T  +  t_hi . [s'_hi ; s'_lo]^T     (N = 128, K = 128 + 64)
//     DB  = t_lo . s'_hi^T                                          (N = 64,  K = 64)
//   z_c = tau (DA[c] + DA[64 + c] + DB[c]) - lambda H_c for eligible chunks, else -inf.
//   Two accumulator sets (192 columns each) let the epilogue of head h overlap the MMAs of
//   head h + 1; the epilogue writes the head's scores and keeps the group maximum zeta.
// Warp roles (384 threads): warp 0 issues the MMAs (warp-collective), warp 1 the TMA loads,
// warps 4-11 read the accumulators (TMEM lane quarter = warp % 4, one query row per thread,
// warps 4-7 chunks 0-31 of the tile, warps 8-11 chunks 32-63).
// Every wait is bounded; after a timeout the kernel records RDL_ERR_TIMEOUT, every role
// stops, the MMAs in flight drain, the last TMA loads land, tensor memory is freed.
#pragma once
#include "common.cuh"
#include "tc.cuh"

namespace rdl {

constexpr int ZT_ROWS = 128, ZT_CH = 64, ZT_THREADS = 384;
constexpr int ZT_OFF_T = 0;                               // [t_hi | t_lo][128 rows][128 B]
constexpr int ZT_OFF_ST = 32768;                          // stage s at + ZT_STAGE s
constexpr int ZT_STAGE = 81920;                           // q 32 KB, s 32 KB, s' 16 KB
constexpr int ZT_OFF_BAR = ZT_OFF_ST + 2 * ZT_STAGE;
constexpr int ZT_OFF_H = ZT_OFF_BAR + 256;                // entropies [8 heads][64] fp32
constexpr int ZT_OFF_P = ZT_OFF_H + 8 * ZT_CH * 4;        // positions [128] int
constexpr int ZT_SMEM = ZT_OFF_P + ZT_ROWS * 4 + 1024;    // + alignment slack
static_assert(ZT_SMEM <= 227 * 1024, "shared memory");

// MODE 0: writes every per-head score (z_all) and the group maximum (zeta);
// MODE 1: writes the group maximum only;
// MODE 2: given the selection idx (ascending per row and group), writes the per-head scores of
//         the selected chunks that fall in the CTA's chunk tile into z_sel.
template <int MODE>
__global__ void __launch_bounds__(ZT_THREADS, 1)
    zeta_tc_kernel(const __grid_constant__ CUtensorMap qmap, const __grid_constant__ CUtensorMap smap,
                   const __grid_constant__ CUtensorMap spmap, const __grid_constant__ CUtensorMap tmap,
                   const int32_t* __restrict__ q_pos, const float* __restrict__ entropy, int Lq, int L, int Hq,
                   int Hkv, int w, float lambda, float* __restrict__ z_all, float* __restrict__ zeta,
                   const int32_t* __restrict__ idx, int K, float* __restrict__ z_sel) {
  constexpr int D = 128;
  extern __shared__ unsigned char zt_raw[];
  unsigned char* sm = zt_raw + ((1024u - (smem_u32(zt_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + ZT_OFF_BAR);
  uint64_t* tload = bars;          // residual rows landed
  uint64_t* full = bars + 1;       // [2] a head's q / s / s' tiles landed
  uint64_t* empty = bars + 3;      // [2] stage consumed (commit)
  uint64_t* afull = bars + 5;      // [2] accumulator set written (commit)
  uint64_t* aempty = bars + 7;     // [2] accumulator set read (8 epilogue warps)
  uint64_t* mdone = bars + 9;      // every MMA of the issuer complete
  uint32_t* tslot = reinterpret_cast<uint32_t*>(bars + 10);
  int* abort_f = reinterpret_cast<int*>(tslot + 1);
  float* Hs = reinterpret_cast<float*>(sm + ZT_OFF_H);
  int* Ps = reinterpret_cast<int*>(sm + ZT_OFF_P);

  const int C = L / S, G = Hq / Hkv;
  const int bg = blockIdx.z, b = bg / Hkv, g = bg % Hkv;
  const int i0 = blockIdx.y * ZT_ROWS, c0 = blockIdx.x * ZT_CH;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float tau = rsqrtf((float)D);

  if (tid == 0) {
    tc::mbar_init(tload, 1);
    for (int j = 0; j < 2; ++j) {
      tc::mbar_init(&full[j], 1);
      tc::mbar_init(&empty[j], 1);
      tc::mbar_init(&afull[j], 1);
      tc::mbar_init(&aempty[j], 8);
    }
    tc::mbar_init(mdone, 1);
    *abort_f = 0;
    tc::mbar_fence_init();
  }
  if (tid < ZT_ROWS) {
    const int i = i0 + tid;
    Ps[tid] = i < Lq ? (q_pos ? q_pos[(size_t)b * Lq + i] : i) : INT_MIN;
  }
  for (int e = tid; e < G * ZT_CH; e += ZT_THREADS) {
    const int hl = e / ZT_CH, cc = e % ZT_CH, c = c0 + cc;
    Hs[hl * ZT_CH + cc] = c < C ? entropy[(size_t)(b * Hq + g * G + hl) * C + c] : 0.f;
  }
  if (warp == 0) {
    tc::tmem_alloc(tslot, 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tslot;

  if (warp == 1) {
    // ---------------- TMA producer
    if (lane == 0) {
      tc::mbar_arrive_expect_tx(tload, 32768u);
      tc::tma_load_3d(sm + ZT_OFF_T, &tmap, 0, b * Lq + i0, 0, tload);
      int n_issued = 0;
      for (int hl = 0; hl < G; ++hl) {
        const int st = hl & 1, n = hl >> 1;
        if ((n > 0 && !tc::mbar_wait(&empty[st], (unsigned)(n - 1) & 1u)) || *(volatile int*)abort_f) {
          *(volatile int*)abort_f = 1;
          break;
        }
        unsigned char* stg = sm + ZT_OFF_ST + st * ZT_STAGE;
        const int h = g * G + hl, srow = (b * Hq + h) * C + c0;
        tc::mbar_arrive_expect_tx(&full[st], (unsigned)ZT_STAGE);
        tc::tma_load_4d(stg, &qmap, 0, b * Lq + i0, 0, h, &full[st]);
        tc::tma_load_4d(stg + 32768, &smap, 0, srow, 0, 0, &full[st]);
        tc::tma_load_3d(stg + 65536, &spmap, 0, srow, 0, &full[st]);
        ++n_issued;
      }
      // the last loads issued into each stage have landed before the CTA may exit
      for (int x = max(0, n_issued - 2); x < n_issued; ++x) (void)tc::mbar_wait(&full[x & 1], (unsigned)(x >> 1) & 1u);
      (void)tc::mbar_wait(tload, 0);
    }
    __syncwarp();
  } else if (warp == 0) {
    // ---------------- MMA issuer (warp-collective, one elected lane issues)
    const uint32_t id128 = tc::idesc_bf16(128, 128, false, false), id64 = tc::idesc_bf16(128, 64, false, false);
    const uint64_t dT = tc::sdesc(smem_u32(sm + ZT_OFF_T), 16, 1024);
    auto wait_all = [&](uint64_t* bar, unsigned ph) -> bool {
      const bool r = tc::mbar_wait(bar, ph) && !*(volatile int*)abort_f;
      return __all_sync(0xffffffffu, r);
    };
    bool ok = wait_all(tload, 0), issued = false;
    for (int hl = 0; hl < G && ok; ++hl) {
      const int st = hl & 1, hb = hl & 1;
      if (!wait_all(&full[st], (unsigned)(hl >> 1) & 1u) || !wait_all(&aempty[hb], ((unsigned)(hl >> 1) & 1u) ^ 1u)) {
        ok = false;
        break;
      }
      tc::tc_fence_after();
      const uint32_t stg = smem_u32(sm + ZT_OFF_ST + st * ZT_STAGE);
      const uint64_t dq = tc::sdesc(stg, 16, 1024), ds = tc::sdesc(stg + 32768, 16, 1024),
                     dsp = tc::sdesc(stg + 65536, 16, 1024);
      const uint32_t DA = tbase + (uint32_t)(192 * hb), DB = DA + 128u;
      // q . [s_hi ; s_lo]: column halves j of q and of the chunk rows are 16 KB apart
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int k = 0; k < 4; ++k)
          tc::mma_bf16_ss_warp(DA, dq + (uint64_t)(j * 1024 + 2 * k), ds + (uint64_t)(j * 1024 + 2 * k), id128,
                               (j | k) != 0);
      // t_hi . [s'_hi ; s'_lo] into the same set, t_lo . s'_hi into DB
#pragma unroll
      for (int k = 0; k < 4; ++k) tc::mma_bf16_ss_warp(DA, dT + (uint64_t)(2 * k), dsp + (uint64_t)(2 * k), id128, true);
#pragma unroll
      for (int k = 0; k < 4; ++k)
        tc::mma_bf16_ss_warp(DB, dT + (uint64_t)(1024 + 2 * k), dsp + (uint64_t)(2 * k), id64, k != 0);
      tc::mma_commit_warp(&afull[hb]);
      tc::mma_commit_warp(&empty[st]);
      issued = true;
    }
    if (!ok && lane == 0) *(volatile int*)abort_f = 1;
    if (issued) tc::mma_commit_warp(mdone); else tc::mbar_arrive_warp(mdone);
    (void)tc::mbar_wait(mdone, 0);
    __syncwarp();
  } else if (warp >= 4 && warp < 12) {
    // ---------------- epilogue: row r of the tile, chunks 32 hf .. 32 hf + 31
    const int quad = warp & 3, hf = (warp - 4) >> 2, r = 32 * quad + lane, i = i0 + r;
    const int p = Ps[r];
    const int cb = c0 + 32 * hf;
    const uint32_t lrow = tc::taddr(tbase, 32 * quad, 0);
    auto wait_all = [&](uint64_t* bar, unsigned ph) -> bool {
      const bool rr = tc::mbar_wait(bar, ph) && !*(volatile int*)abort_f;
      return __all_sync(0xffffffffu, rr);
    };
    // eligibility of the 32 chunks for this row, as a bit mask
    uint32_t em = 0u;
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (cb + e < C && chunk_eligible(cb + e, p, w)) em |= 1u << e;
    float zmax[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) zmax[e] = -INFINITY;
    const bool vec = (C & 3) == 0 && cb + 32 <= C;
    bool ok = true;
    // MODE 2: the row's selection as a mask over chunks cb .. cb + 31 (bit e: chunk cb + e is
    // selected) and k0, the number of selected chunks below cb, so that chunk cb + e sits in
    // slot k0 + popc(sel & ((1 << e) - 1)) of the ascending list; the row's K indices are
    // loaded at once (K <= 64)
    uint32_t sel = 0u;
    int k0 = 0;
    if (MODE == 2 && i < Lq) {
      const int32_t* irow = idx + ((size_t)bg * Lq + i) * K;
      int v[64];
      if ((K & 3) == 0) {
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int4 q4 = 4 * u < K ? __ldg(reinterpret_cast<const int4*>(irow) + u) : make_int4(-1, -1, -1, -1);
          v[4 * u] = q4.x; v[4 * u + 1] = q4.y; v[4 * u + 2] = q4.z; v[4 * u + 3] = q4.w;
        }
      } else {
#pragma unroll
        for (int u = 0; u < 64; ++u) v[u] = u < K ? __ldg(irow + u) : -1;
      }
#pragma unroll
      for (int u = 0; u < 64; ++u) {
        const int c = v[u];
        if (c >= 0 && c < cb) ++k0;
        if (c >= cb && c < cb + 32) sel |= 1u << (c - cb);
      }
    }
    for (int hl = 0; hl < G; ++hl) {
      const int hb = hl & 1;
      if (!wait_all(&afull[hb], (unsigned)(hl >> 1) & 1u)) { ok = false; break; }
      tc::tc_fence_after();
      float v1[32], v2[32], v3[32];
      tc::tmem_ld32(lrow + (uint32_t)(192 * hb + 32 * hf), v1);
      tc::tmem_ld32(lrow + (uint32_t)(192 * hb + 64 + 32 * hf), v2);
      tc::tmem_ld32(lrow + (uint32_t)(192 * hb + 128 + 32 * hf), v3);
      tc::tmem_wait_ld();
      tc::tc_fence_before();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&aempty[hb]);
      const float* hrow = Hs + hl * ZT_CH + 32 * hf;
      float* z = v1;                     // the scores replace the first term in place
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        z[e] = ((em >> e) & 1u) ? tau * (v1[e] + (v2[e] + v3[e])) - lambda * hrow[e] : -INFINITY;
        zmax[e] = fmaxf(zmax[e], z[e]);
      }
      if (MODE == 2) {
        if (sel) {
          float* zs = z_sel + ((size_t)(b * Hq + g * G + hl) * Lq + i) * K + k0;
#pragma unroll
          for (int x = 0; x < 32; ++x)
            if ((sel >> x) & 1u) zs[__popc(sel & ((1u << x) - 1u))] = z[x];
        }
      } else if (MODE == 0 && i < Lq) {
        float* zr = z_all + ((size_t)(b * Hq + g * G + hl) * Lq + i) * C + cb;
        if (vec) {
#pragma unroll
          for (int e = 0; e < 32; e += 4) *reinterpret_cast<float4*>(zr + e) = make_float4(z[e], z[e + 1], z[e + 2], z[e + 3]);
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e)
            if (cb + e < C) zr[e] = z[e];
        }
      }
    }
    if (MODE != 2 && ok && i < Lq) {
      float* zr = zeta + ((size_t)(b * Hkv + g) * Lq + i) * C + cb;
      if (vec) {
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(zr + e) = make_float4(zmax[e], zmax[e + 1], zmax[e + 2], zmax[e + 3]);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (cb + e < C) zr[e] = zmax[e];
      }
    }
    if (!ok && lane == 0) *(volatile int*)abort_f = 1;
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) tc::tmem_dealloc(tbase, 512);
}

}  // namespace rdl

namespace rdl {

}  // namespace rdl
