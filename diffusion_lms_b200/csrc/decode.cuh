// Route layer and sliding window for decode blocks: a few query rows (at most 64 per
// sequence) against a long cached context.  Same definitions as the prefill kernels
// (Prefilling-dLLM v2, Figure 3 caption; Table 3 for the window and the remote chunks),
// organised for this shape, where the bytes that must come from HBM are the cached
// summaries (fp32, read once) and the K/V slabs of the selected chunks:
//
//   dec_t_kernel      t = x W_down: 8 CTAs, each contracts one slice of the hidden size on
//                     tensor cores and writes its partial; the scorer sums the partials in
//                     a fixed order.
//   dec_score_kernel  CTA = (batch, query head, chunk range).  Before its dependency wait it
//                     starts TMA loads of its summary rows into shared memory (and pulls the
//                     rest into L2), so the one pass over the summaries overlaps the
//                     residual.  Then q_res = q + t W_up for its head and the split-bf16
//                     score z = tau q_res.s - lambda H on tcgen05 tensor cores (summary rows
//                     as the M = 128 operand, accumulators in tensor memory).
//   dec_topk_kernel   CTA = (batch, query row, KV group): zeta = max over the group's heads,
//                     exact top-K (candidate filter, radix select on heavy ties), per-head
//                     scores of the selected chunks.
//   dec_attn_kernel   chunk-major: the CTAs of a (batch, group) split the 64-key slabs that
//                     some row needs (a selected chunk or a window slab) into contiguous
//                     ranges of equal work, stream each slab's K/V once through a TMA ring
//                     and compute every task on it (two rows per warp on tensor cores).
//   dec_comb_kernel   one partition per (row, head): Z = e^lambda_loc + sum_c e^{z_c} and
//                     o = (e^lambda_loc o_loc + sum_c e^{z_c} o_c) / Z, in a fixed order.
//
// The kernels of one call are chained with programmatic dependent launch: every kernel
// waits (griddepcontrol.wait) before it touches anything an earlier kernel writes (read
// after write) and before its first store to a buffer an earlier kernel may still read
// (write after read: two calls in a row on one workspace), and allows its dependent to
// launch only after that wait, so the early start of a dependent never reads data older
// than the call's own inputs nor overwrites data its predecessors still need.  Work that
// reads only inputs of the call and writes only shared memory may run before the wait.
#pragma once
#include "common.cuh"
#include "tc.cuh"
#include "score.cuh"

// Phase markers: empty unless a build defines them (kernel id, slot).
#ifndef RDL_TRACE_POINT
#define RDL_TRACE_POINT(kernel, slot)
#endif

namespace rdl {
namespace dec {

__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }

// fp32 pair -> (hi, lo) packed bf16 pairs with x = hi + lo to ~2^-17 relative.
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat16 h0 = __float2bfloat16_rn(x0), h1 = __float2bfloat16_rn(x1);
  const __nv_bfloat162 hh = __halves2bfloat162(h0, h1);
  const __nv_bfloat162 ll = __floats2bfloat162_rn(x0 - __bfloat162float(h0), x1 - __bfloat162float(h1));
  hi = *reinterpret_cast<const uint32_t*>(&hh);
  lo = *reinterpret_cast<const uint32_t*>(&ll);
}

__device__ __forceinline__ float2 lds_f2(uint32_t addr) {
  float2 v;
  asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];\n" : "=f"(v.x), "=f"(v.y) : "r"(addr));
  return v;
}

// =====================================================================================
// dec_t_kernel: partial t of a hidden slice, tp[rank][M, r] = x[M, slice] W_down[slice, r]
// (bf16 inputs, exact products, fp32 sums).  8 CTAs; CTA `rank` owns hidden slice
// [rank*slice, rank*slice + slice).  The scorer sums the 8 partials in rank order (the
// same result on every run); no cross-CTA barrier, which under the scorer's early summary
// stream measured 2-3 us.
// =====================================================================================
constexpr int TK_CL = 8;
constexpr int TK_KMAX = 512;                                // hidden columns per load batch

// shared memory of dec_t_kernel for `rows` (multiple of 16) query rows, rank r and a batch
// of kc hidden columns (multiple of 64): per 64-column block, x [rows][128 B] and
// W_down [64][128 B] per 64 columns of r (TMA boxes, 128-byte swizzle).
__host__ __device__ inline int tk_smem(int rows, int r, int kc) {
  return 1024 + (kc / 64) * (rows * 128 + (r / 64) * 8192) + 16;
}

__global__ void __launch_bounds__(256)
    dec_t_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap wmap, int M,
                 int D, int r, int kc, float* __restrict__ tp) {
  extern __shared__ unsigned char tk_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(tk_raw) + 1023) & ~uintptr_t(1023));
  RDL_TRACE_POINT(0, 0);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int Mt = (M + 15) >> 4, rows = Mt * 16;
  const int nkb = kc / 64, nnb = r / 64;
  const int xblk = rows * 128, wblk = nnb * 8192;
  unsigned char* xs = base;                                    // [nkb][rows][128 B]
  unsigned char* ws = xs + nkb * xblk;                         // [nkb][nnb][64][128 B]
  uint64_t* bar = reinterpret_cast<uint64_t*>(ws + nkb * wblk);
  if (tid == 0) {
    tc::mbar_init(bar, 1);
    tc::mbar_fence_init();
  }
  __syncthreads();
  grid_dep_wait();
  grid_dep_launch();
  RDL_TRACE_POINT(0, 1);
  const int rank = blockIdx.x;
  const int slice = ((D + TK_CL * 64 - 1) / (TK_CL * 64)) * 64;
  const int k0 = min(D, rank * slice), k1 = min(D, k0 + slice);
  const int npairs = r / 16, ntask = Mt * npairs;
  float acc[4][2][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int n = 0; n < 2; ++n) acc[a][n][0] = acc[a][n][1] = acc[a][n][2] = acc[a][n][3] = 0.f;

  unsigned phase = 0;
  for (int kb = k0; kb < k1; kb += kc) {
    const int nb = min(kc, k1 - kb) / 64;                      // 64-column blocks in this batch
    if (tid == 0) {
      tc::mbar_arrive_expect_tx(bar, (unsigned)(nb * (xblk + wblk)));
      for (int j = 0; j < nb; ++j) {
        tc::tma_load_2d(xs + j * xblk, &xmap, kb + 64 * j, 0, bar);
        for (int n = 0; n < nnb; ++n) tc::tma_load_2d(ws + j * wblk + n * 8192, &wmap, 64 * n, kb + 64 * j, bar);
      }
    }
    if (!tc::mbar_wait(bar, phase)) break;
    phase ^= 1u;
    RDL_TRACE_POINT(0, 2);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int task = warp + 8 * a;
      if (task >= ntask) break;
      const int mt = task / npairs, np = task % npairs;
      for (int ks = 0; ks < nb * 4; ++ks) {
        const unsigned char* xb = xs + (ks >> 2) * xblk;
        const unsigned char* wb = ws + (ks >> 2) * wblk + (np >> 2) * 8192;
        const int kq = (ks & 3) * 16;
        uint32_t af[4];
        const int ra = mt * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        ldsm_x4(smem_u32(xb + tc::sw128(ra, kq + 8 * (lane >> 4))), af[0], af[1], af[2], af[3]);
        uint32_t b0, b1, b2, b3;
        const int mi = lane >> 3, kk = kq + 8 * (mi & 1) + (lane & 7), nn = ((2 * np) & 7) * 8 + 8 * (mi >> 1);
        ldsm_x4_t(smem_u32(wb + tc::sw128(kk, nn)), b0, b1, b2, b3);
        mma_bf16(acc[a][0], af, b0, b1);
        mma_bf16(acc[a][1], af, b2, b3);
      }
    }
    __syncthreads();
  }
  RDL_TRACE_POINT(0, 3);
  // this CTA's partial straight from the accumulators
  const int gq = lane >> 2, tq = lane & 3;
  float* tr = tp + (size_t)rank * M * r;
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int task = warp + 8 * a;
    if (task >= ntask) break;
    const int mt = task / npairs, np = task % npairs;
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int row = mt * 16 + gq + 8 * hr;
      if (row >= M) continue;
#pragma unroll
      for (int n = 0; n < 2; ++n) {
        const int col = (2 * np + n) * 8 + 2 * tq;
        *reinterpret_cast<float2*>(tr + (size_t)row * r + col) = make_float2(acc[a][n][2 * hr], acc[a][n][2 * hr + 1]);
      }
    }
  }
  RDL_TRACE_POINT(0, 4);
}

// =====================================================================================
// dec_score_kernel: CTA = (chunk range, query head h, batch b); 16 warps.
// MT = m-tiles of 16 query rows (NR = 16*MT >= Lq rows).
// The score tile of one box is D[chunk][row] = s_c . q_res on the 5th-generation tensor
// cores: M = 128 summary rows straight from the TMA ring (K-major, 128-byte swizzle), K = d,
// three bf16 split terms: s_hi x [q_hi; q_lo] (N = 2 NR, one operand read for two terms) and
// s_lo x q_hi (N = NR), in tensor memory (two accumulator sets, so the epilogue of box n
// overlaps the MMAs of box n + 1).
// Shared memory:
//   ring   nstg stages of SC_BOXR summary rows; split layout: [4 segments][SC_BOXR][128 B]
//          (hi 0-63, hi 64-127, lo 0-63, lo 64-127); fp32 layout: [4 slices][SC_BOXR][32 fp32],
//          rewritten in place to [32 bf16 hi | 32 bf16 lo] per slice row once landed
//   qsp    q_res split into bf16 hi/lo, K-major with the 128-byte swizzle:
//          [2 K segments (columns 0-63, 64-127)][q_hi rows 0..NR-1, q_lo rows][128 B]
//   wup    W_up columns of head h: [r][128] bf16, unit-swizzled (ldmatrix.trans)
//   ts     t rows: [NR][r + 8] fp32
//   hs     entropies of the range; wl/wh: per-row window chunk range (not eligible)
// Warp roles after the residual: warps 0 and 2 issue the MMAs of the two accumulators
// (warp-collective), warp 1 refills the ring (one thread), the epilogue warps read the
// accumulators (TMEM lane quarter = warp % 4) and store the scores: warps 4-11 (two row
// halves) for split summaries, warps 4-7 for fp32 ones, whose boxes warps 8-15 convert.
// =====================================================================================
constexpr int SC_WARPS = 16;
constexpr int SC_BOXR = 128;                 // summary rows per box = MMA M
constexpr int SC_BOX_BYTES = SC_BOXR * 512;
__host__ __device__ constexpr int sc_epi_warps(bool split) { return split ? 8 : 4; }
struct ScoreSmem {
  int ring, qsp, wup, ts, hs, win, bar, total;
};
__host__ __device__ inline ScoreSmem score_smem(int MT, int r, int nstg, int ncr) {
  ScoreSmem s{};
  const int NR = 16 * MT;
  int off = 0;
  s.ring = off; off += nstg * SC_BOX_BYTES;
  s.qsp = off;  off += 4 * NR * 128;
  s.wup = off;  off += (r > 0 ? r : 1) * 256;
  s.ts = off;   off += NR * (r + 8) * 4;
  s.hs = off;   off += ((ncr + 3) & ~3) * 4;
  s.win = off;  off += 2 * NR * 4;
  s.bar = off;  off += 8 * (3 * nstg + 5) + 16;
  s.total = off + 1024;       // slack for aligning the base to 1024 bytes
  return s;
}

// byte offset of column col (0..255: hi 0-127, lo 128-255) of row `row` in the qsp tile
// (NR a multiple of 8, so the swizzle row r2 % 8 equals row % 8)
__device__ __forceinline__ uint32_t qsp_off(int NR, int row, int col) {
  const int ksg = (col & 127) >> 6, r2 = (col >> 7) * NR + row, within = col & 63;
  return (uint32_t)(ksg * 2 * NR * 128 + r2 * 128 + (((within >> 3) ^ (r2 & 7)) << 4) + (within & 7) * 2);
}

template <int MT, bool SPLIT>
__global__ void __launch_bounds__(SC_WARPS * 32, 1)
    dec_score_kernel(const __grid_constant__ CUtensorMap smap, const float* __restrict__ smap_base,
                     const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ q_pos,
                     const float* __restrict__ t, const __nv_bfloat16* __restrict__ w_up,
                     const float* __restrict__ entropy, int Lq, int L, int Hq, int r, int w, float tau,
                     float lambda, int ncr, int nstg, float* __restrict__ z_all) {
  constexpr int D = 128;
  constexpr int NT = SC_WARPS * 32;
  constexpr int NR = 16 * MT;
  constexpr int NG = SC_WARPS / MT;           // warps per m-tile in the residual (n-groups)
  constexpr int NPW = 16 / NG;                // residual n-tiles (of 8 columns) per warp
  // two accumulator sets of 3 NR columns: [s_hi.q_hi | s_hi.q_lo] (2 NR) and s_lo.q_hi (NR)
  constexpr uint32_t TCOLS = 6 * NR <= 128 ? 128 : (6 * NR <= 256 ? 256 : 512);
  extern __shared__ unsigned char sc_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(sc_raw) + 1023) & ~uintptr_t(1023));
  const ScoreSmem L_ = score_smem(MT, r, nstg, ncr);
  unsigned char* ring = base + L_.ring;
  unsigned char* qsp = base + L_.qsp;
  unsigned char* wup = base + L_.wup;
  float* ts = reinterpret_cast<float*>(base + L_.ts);
  float* hs = reinterpret_cast<float*>(base + L_.hs);
  int* wl = reinterpret_cast<int*>(base + L_.win);
  int* wh = wl + NR;
  uint64_t* full = reinterpret_cast<uint64_t*>(base + L_.bar);
  uint64_t* empty = full + nstg;
  uint64_t* conv = empty + nstg;
  uint64_t* tfull = conv + nstg;
  uint64_t* tempty = tfull + 2;
  uint64_t* mdone = tempty + 2;
  uint32_t* tslot = reinterpret_cast<uint32_t*>(mdone + 1);
  int* abort_f = reinterpret_cast<int*>(tslot + 1);
  RDL_TRACE_POINT(1, 0);

  const int C = L / S;
  const int b = blockIdx.z, h = blockIdx.y;
  const int c0 = blockIdx.x * ncr, c1 = min(C, c0 + ncr);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int mw = warp % MT, ng = warp / MT;
  if (c0 >= C) {
    grid_dep_wait();
    return;
  }
  const int nb = (c1 - c0 + SC_BOXR - 1) / SC_BOXR;
  const size_t srow0 = (size_t)(b * Hq + h) * C + c0;
  // ---- prologue: only TMA and cp.async.cg loads of inputs (no kernel of this call writes
  // them, and this kernel is launched early only behind dec_t_kernel, which has waited)
  constexpr int EW = sc_epi_warps(SPLIT);
  const int npro = min(nb, nstg);     // boxes loaded before the dependency wait
  if (tid == 0) {
    for (int st = 0; st < nstg; ++st) {
      tc::mbar_init(&full[st], 1);
      tc::mbar_init(&empty[st], 2);
      tc::mbar_init(&conv[st], 8);
    }
    for (int j = 0; j < 2; ++j) {
      tc::mbar_init(&tfull[j], 2);
      tc::mbar_init(&tempty[j], EW);
    }
    tc::mbar_init(mdone, 2);
    *abort_f = 0;
    tc::mbar_fence_init();
    for (int bx = 0; bx < npro; ++bx) {
      tc::mbar_arrive_expect_tx(&full[bx], (unsigned)SC_BOX_BYTES);
      tc::tma_load_3d(ring + bx * SC_BOX_BYTES, &smap, 0, (int)(srow0 + (size_t)bx * SC_BOXR), 0, &full[bx]);
    }
  }
  if (warp == 0) {
    __syncwarp();
    tc::tmem_alloc(tslot, TCOLS);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tbase = *tslot;
  int n_issued = npro;                // boxes issued (prologue, then refills by thread 32)
  for (int e = tid; e < r * 16; e += NT) {
    const int kk = e >> 4, u = e & 15;
    cp_async16(smem_u32(wup + kk * 256 + ((u ^ (kk & 7)) << 4)), w_up + (size_t)kk * Hq * D + h * D + u * 8);
  }
  cp_async_commit();
  // the q values this thread adds to its residual fragment (rows row0/row1, NPW n-tiles)
  __nv_bfloat162 qv[NPW][2];
  {
    const int row0 = mw * 16 + gq;
#pragma unroll
    for (int n = 0; n < NPW; ++n) {
      const int col = (ng * NPW + n) * 8 + 2 * tq;
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int row = row0 + 8 * hr;
        qv[n][hr] = row < Lq ? *reinterpret_cast<const __nv_bfloat162*>(q + ((size_t)(b * Lq + row) * Hq + h) * D + col)
                             : __floats2bfloat162_rn(0.f, 0.f);
      }
    }
  }
  for (int j = tid; j < c1 - c0; j += NT) hs[j] = __ldcg(entropy + (size_t)(b * Hq + h) * C + c0 + j);
  if (tid < NR) {
    // window chunk range of row tid: chunks wl..wh are not eligible (empty when wl > wh)
    const int p = tid < Lq ? (q_pos ? __ldcg(q_pos + (size_t)b * Lq + tid) : tid) : INT_MIN;
    if (w < 0 || p == INT_MIN) {
      wl[tid] = 1;
      wh[tid] = 0;
    } else {
      wl[tid] = p - w <= 0 ? INT_MIN : (p - w) / S;
      wh[tid] = (p + w) / S;
    }
  }
  // rows beyond the ring: pulled into L2 now, loaded into the ring when a stage frees
  for (int bx = nstg + warp; bx < nb; bx += SC_WARPS) {
    const char* src = reinterpret_cast<const char*>(smap_base) + (srow0 + (size_t)bx * SC_BOXR) * 512;
    const int bytes = min(SC_BOXR, (c1 - c0) - bx * SC_BOXR) * 512;
    for (int off = lane * 4096; off < bytes; off += 32 * 4096)
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(src + off), "r"(min(4096, bytes - off))
                   : "memory");
  }

  grid_dep_wait();      // t is written by dec_t_kernel
  grid_dep_launch();
  RDL_TRACE_POINT(1, 1);
  if (r > 0) {
    // t rows = the TK_CL partials of dec_t_kernel summed in rank order
    const int nu = r / 4;                       // 16-byte units per t row
    const size_t pstride = (size_t)gridDim.z * Lq * r;
    for (int e = tid; e < Lq * nu; e += NT) {
      const int i = e / nu, u = e % nu;
      const float4* src = reinterpret_cast<const float4*>(t + (size_t)(b * Lq + i) * r + u * 4);
      float4 pv[TK_CL];
#pragma unroll
      for (int k = 0; k < TK_CL; ++k) pv[k] = __ldcg(src + k * (pstride / 4));
      float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int k = 0; k < TK_CL; ++k) {
        acc.x += pv[k].x;
        acc.y += pv[k].y;
        acc.z += pv[k].z;
        acc.w += pv[k].w;
      }
      *reinterpret_cast<float4*>(ts + i * (r + 8) + u * 4) = acc;
    }
  }
  cp_async_commit();

  // ---- q_res = q + t W_up for this warp's m-tile and n-group (tensor cores, t split),
  // written straight into the split hi/lo operand tile
  {
    float ua[NPW][4];
#pragma unroll
    for (int n = 0; n < NPW; ++n) ua[n][0] = ua[n][1] = ua[n][2] = ua[n][3] = 0.f;
    const int row0 = mw * 16 + gq, row1 = row0 + 8;
    cp_async_wait<0>();
    __syncthreads();
    RDL_TRACE_POINT(1, 2);
    for (int kk = 0; kk < r / 16; ++kk) {
      uint32_t ahi[4], alo[4];
      {
        const int ca = 16 * kk + 2 * tq, rs = r + 8;
        const float2 z2 = make_float2(0.f, 0.f);
        const float2 v0 = row0 < Lq ? *reinterpret_cast<const float2*>(ts + row0 * rs + ca) : z2;
        const float2 v1 = row1 < Lq ? *reinterpret_cast<const float2*>(ts + row1 * rs + ca) : z2;
        const float2 v2 = row0 < Lq ? *reinterpret_cast<const float2*>(ts + row0 * rs + ca + 8) : z2;
        const float2 v3 = row1 < Lq ? *reinterpret_cast<const float2*>(ts + row1 * rs + ca + 8) : z2;
        split2(v0.x, v0.y, ahi[0], alo[0]);
        split2(v1.x, v1.y, ahi[1], alo[1]);
        split2(v2.x, v2.y, ahi[2], alo[2]);
        split2(v3.x, v3.y, ahi[3], alo[3]);
      }
#pragma unroll
      for (int n = 0; n < NPW; n += 2) {
        const int nt = ng * NPW + n;
        uint32_t b0, b1, b2, b3;
        const int mi = lane >> 3, k = 16 * kk + 8 * (mi & 1) + (lane & 7), un = nt + (mi >> 1);
        ldsm_x4_t(smem_u32(wup + k * 256 + ((un ^ (k & 7)) << 4)), b0, b1, b2, b3);
        mma_bf16(ua[n], ahi, b0, b1);
        mma_bf16(ua[n], alo, b0, b1);
        mma_bf16(ua[n + 1], ahi, b2, b3);
        mma_bf16(ua[n + 1], alo, b2, b3);
      }
    }
#pragma unroll
    for (int n = 0; n < NPW; ++n) {
      const int col = (ng * NPW + n) * 8 + 2 * tq;
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int row = mw * 16 + gq + 8 * hr;
        const float2 qf = __bfloat1622float2(qv[n][hr]);
        uint32_t hi, lo;
        split2(qf.x + ua[n][2 * hr], qf.y + ua[n][2 * hr + 1], hi, lo);
        *reinterpret_cast<uint32_t*>(qsp + qsp_off(NR, row, col)) = hi;
        *reinterpret_cast<uint32_t*>(qsp + qsp_off(NR, row, 128 + col)) = lo;
      }
    }
  }
  tc::fence_proxy_async();            // the operand tile is read by the tensor cores
  __syncthreads();
  RDL_TRACE_POINT(1, 3);

  if (warp == 0 || warp == 2) {
    // ---------------- MMA issuers (warp-collective, one elected lane issues): warp 0 the
    // s_hi x [q_hi; q_lo] accumulator, warp 2 the s_lo x q_hi one
    const bool hi_set = warp == 0;
    const uint32_t idesc = hi_set ? tc::idesc_bf16(128, 2 * NR, false, false) : tc::idesc_bf16(128, NR, false, false);
    const uint64_t dq0 = tc::sdesc(smem_u32(qsp), 16, 1024);
    const uint64_t qks = (uint64_t)((2 * NR * 128) >> 4);        // K segment of the q tile
    const uint64_t aseg = (uint64_t)((SC_BOXR * 128) >> 4);      // segment of a box
    bool issued = false;
    for (int bx = 0; bx < nb; ++bx) {
      const int st = bx % nstg, buf = bx & 1;
      const unsigned ph = (unsigned)(bx / nstg) & 1u;
      const bool ok = tc::mbar_wait(SPLIT ? &full[st] : &conv[st], ph) &&
                      tc::mbar_wait(&tempty[buf], ((unsigned)(bx >> 1) & 1u) ^ 1u) && !*(volatile int*)abort_f;
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) *(volatile int*)abort_f = 1;
        break;
      }
      if (bx == 0) RDL_TRACE_POINT(1, 4);
      if (bx == 1) RDL_TRACE_POINT(1, 6);
      if (bx == nb - 1) RDL_TRACE_POINT(1, 7);
      tc::tc_fence_after();
      const uint64_t da0 = tc::sdesc(smem_u32(ring + st * SC_BOX_BYTES), 16, 1024);
      const uint32_t dt = tbase + (uint32_t)(buf * 3 * NR + (hi_set ? 0 : 2 * NR));
      if (SPLIT) {
        // box segments: 0, 1 = s hi (columns 0-63, 64-127), 2, 3 = s lo
        const int sa = hi_set ? 0 : 2;
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int k = 0; k < 4; ++k)
            tc::mma_bf16_ss_warp(dt, da0 + (sa + j) * aseg + 2 * k, dq0 + j * qks + 2 * k, idesc, (j | k) != 0);
      } else {
        // slice s holds columns 32s..32s+31 as [16 hi | 16 hi | 16 lo | 16 lo] (32 B each)
        const int ao = hi_set ? 0 : 4;
#pragma unroll
        for (int sl = 0; sl < 4; ++sl)
#pragma unroll
          for (int k = 0; k < 2; ++k) {
            const uint64_t bq = dq0 + (uint64_t)(sl >> 1) * qks + (uint64_t)((sl & 1) * 4 + 2 * k);
            tc::mma_bf16_ss_warp(dt, da0 + sl * aseg + ao + 2 * k, bq, idesc, (sl | k) != 0);
          }
      }
      tc::mma_commit_warp(&tfull[buf]);
      tc::mma_commit_warp(&empty[st]);
      issued = true;
    }
    // every MMA issued has completed before the tensor memory is released
    if (issued) tc::mma_commit_warp(mdone); else tc::mbar_arrive_warp(mdone);
    (void)tc::mbar_wait(mdone, 0);
    __syncwarp();
  } else if (warp == 1) {
    // ---------------- ring refills (the stage's MMAs have completed)
    if (lane == 0) {
      for (int bx = nstg; bx < nb; ++bx) {
        const int st = bx % nstg;
        if (!tc::mbar_wait(&empty[st], (unsigned)(bx / nstg - 1) & 1u) || *(volatile int*)abort_f) {
          *(volatile int*)abort_f = 1;
          break;
        }
        tc::mbar_arrive_expect_tx(&full[st], (unsigned)SC_BOX_BYTES);
        tc::tma_load_3d(ring + st * SC_BOX_BYTES, &smap, 0, (int)(srow0 + (size_t)bx * SC_BOXR), 0, &full[st]);
        ++n_issued;
      }
      // the last box issued into each stage has landed before the CTA may exit
      for (int bx = max(0, n_issued - nstg); bx < n_issued; ++bx)
        (void)tc::mbar_wait(&full[bx % nstg], (unsigned)(bx / nstg) & 1u);
    }
    __syncwarp();
  } else if (warp >= 4 && warp < 4 + EW) {
    // ---------------- epilogue: lanes 32 (warp % 4) .. + 31 of the accumulator = chunks;
    // rows [r0, r0 + RPW) of them
    constexpr int RPW = NR * 4 / EW;
    constexpr int CH = RPW < 16 ? RPW : 16;
    const int quad = warp & 3, r0 = ((warp - 4) >> 2) * RPW;
    // chunks outside [wmin, wmax] are eligible for every row (the usual case: the rows of a
    // block share one narrow window), so the per-row test runs only inside it
    int wmin = INT_MAX, wmax = INT_MIN;
    for (int i = 0; i < Lq; ++i)
      if (wl[i] <= wh[i]) {
        wmin = min(wmin, wl[i]);
        wmax = max(wmax, wh[i]);
      }
    for (int bx = 0; bx < nb; ++bx) {
      const int buf = bx & 1;
      const bool ok = tc::mbar_wait(&tfull[buf], (unsigned)(bx >> 1) & 1u) && !*(volatile int*)abort_f;
      if (!__all_sync(0xffffffffu, ok)) {
        if (lane == 0) *(volatile int*)abort_f = 1;
        break;
      }
      const int c = c0 + bx * SC_BOXR + 32 * quad + lane;
      // eligibility of (row, c) as a bit mask and the entropy term, read before any store
      unsigned long long em = ~0ull;
      if (c >= wmin && c <= wmax) {
        em = 0ull;
        for (int i = 0; i < NR; ++i)
          if (c < wl[i] || c > wh[i]) em |= 1ull << i;
      }
      const float eh = c < c1 ? lambda * hs[c - c0] : 0.f;
      float* zc = z_all + (size_t)(b * Hq + h) * Lq * C + c;
      tc::tc_fence_after();
      const uint32_t ta = tc::taddr(tbase, 32 * quad, buf * 3 * NR);
#pragma unroll
      for (int i0 = r0; i0 < r0 + RPW; i0 += CH) {
        float vh[CH], vl[CH], vs[CH];
        if constexpr (CH == 16) {
          tc::tmem_ld16(ta + i0, vh);
          tc::tmem_ld16(ta + NR + i0, vl);
          tc::tmem_ld16(ta + 2 * NR + i0, vs);
        } else {
          tc::tmem_ld8(ta + i0, vh);
          tc::tmem_ld8(ta + NR + i0, vl);
          tc::tmem_ld8(ta + 2 * NR + i0, vs);
        }
        tc::tmem_wait_ld();
        if (i0 + CH >= r0 + RPW) {
          tc::tc_fence_before();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&tempty[buf]);
        }
        if (c < c1) {
#pragma unroll
          for (int e = 0; e < CH; ++e) {
            const int i = i0 + e;
            if (i >= Lq) break;
            const float acc = vh[e] + (vl[e] + vs[e]);
            __stcg(zc + (size_t)i * C, ((em >> i) & 1ull) ? tau * acc - eh : -INFINITY);
          }
        }
      }
    }
  } else if (!SPLIT && warp >= 8) {
    // ---------------- fp32 boxes: rewrite every 128-byte slice row (32 fp32) in place as
    // 32 bf16 hi terms then 32 bf16 lo terms (x = hi + lo to ~2^-17), keeping the swizzle
    const int ct = tid - 256;
    for (int bx = 0; bx < nb; ++bx) {
      const int st = bx % nstg;
      if (!tc::mbar_wait(&full[st], (unsigned)(bx / nstg) & 1u) || *(volatile int*)abort_f) {
        *(volatile int*)abort_f = 1;
        break;
      }
      unsigned char* stg = ring + st * SC_BOX_BYTES;
      for (int seg = ct; seg < 4 * SC_BOXR; seg += 256) {
        const int rr = seg % SC_BOXR;
        unsigned char* sp = stg + (seg / SC_BOXR) * SC_BOXR * 128 + rr * 128;
        const int sw = rr & 7;
        float4 vv[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) vv[u] = *reinterpret_cast<const float4*>(sp + ((u ^ sw) << 4));
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          split2(vv[u].x, vv[u].y, hi[2 * u], lo[2 * u]);
          split2(vv[u].z, vv[u].w, hi[2 * u + 1], lo[2 * u + 1]);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          *reinterpret_cast<uint4*>(sp + ((u ^ sw) << 4)) = make_uint4(hi[4 * u], hi[4 * u + 1], hi[4 * u + 2], hi[4 * u + 3]);
          *reinterpret_cast<uint4*>(sp + (((4 + u) ^ sw) << 4)) =
              make_uint4(lo[4 * u], lo[4 * u + 1], lo[4 * u + 2], lo[4 * u + 3]);
        }
      }
      tc::fence_proxy_async();
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&conv[st]);
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  if (warp == 0) tc::tmem_dealloc(tbase, TCOLS);
  RDL_TRACE_POINT(1, 5);
}

// =====================================================================================
// dec_topk_kernel: CTA = (query row i, group g, batch b), 256 threads.  The G score rows
// of (i, g) arrive in shared memory in one cp.async batch when C % 4 == 0 and G*C fits
// (ZS = true); otherwise they are read from global memory.
// =====================================================================================
constexpr int DK_MAXZ = 8 * 4096;           // floats of staged score rows

// Top-K of the group max by a candidate filter.  Keys are (order_key(zeta), ~chunk) packed
// in 64 bits, so larger means better with ties to the smaller chunk.  Every warp finds its
// q-th largest key (q = ceil(K / 8)); the smallest of those eight bounds the K-th largest key
// from below (each warp holds q keys at or above its own bound), so every key of the top K is
// among the candidates at or above it.  The candidates (typically a few more than K) are
// ranked exactly; more than DK_MAXCAND of them (heavy ties) falls back to the radix select.
constexpr int DK_MAXCAND = 256;

constexpr int DK_THREADS = 512;
template <bool ZS, int MAXM>
__global__ void __launch_bounds__(DK_THREADS) dec_topk_kernel(const float* __restrict__ z_all,
                                                       const int32_t* __restrict__ q_pos, int Lq, int L,
                                                       int Hq, int Hkv, int K, int32_t* __restrict__ idx,
                                                       float* __restrict__ z_sel) {
  extern __shared__ __align__(128) uint32_t dk_smem[];
  __shared__ unsigned hist[256];
  __shared__ unsigned whist[DK_THREADS / 32][256];
  __shared__ int warp_sums[DK_THREADS / 32];
  __shared__ int sel_s[64];
  __shared__ int bc[3];
  __shared__ unsigned long long wbound[DK_THREADS / 32];
  __shared__ unsigned long long cand[DK_MAXCAND];
  __shared__ int ncand_s;
  __shared__ __align__(8) uint64_t zbar;
  RDL_TRACE_POINT(2, 0);
  const int C = L / S, G = Hq / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int i = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  // the row position is an input of the call (read before the wait: this kernel starts
  // early only behind the scorer, which has waited)
  const int p = q_pos ? __ldcg(q_pos + (size_t)b * Lq + i) : i;
  if (threadIdx.x == 0) {
    tc::mbar_init(&zbar, 1);
    tc::mbar_fence_init();
  }
  __syncthreads();
  grid_dep_wait();
  grid_dep_launch();
  RDL_TRACE_POINT(2, 1);
  uint32_t* keys = dk_smem;                                        // [C]
  float* zs = reinterpret_cast<float*>(dk_smem + ((C + 3) & ~3));  // [G][C] (ZS)
  const float* z0 = z_all + ((size_t)(b * Hq + g * G) * Lq + i) * C;
  const size_t hstride = (size_t)Lq * C;
  int32_t* irow = idx + ((size_t)(b * Hkv + g) * Lq + i) * K;
  if (is_mask_slot(p)) {
    for (int e = tid; e < K * G; e += DK_THREADS) {
      const int k = e % K, hl = e / K;
      if (hl == 0) irow[k] = -1;
      z_sel[((size_t)(b * Hq + g * G + hl) * Lq + i) * K + k] = -INFINITY;
    }
    return;
  }
  if (ZS) {
    // the group's G score rows: G bulk copies on one barrier
    if (tid == 0) {
      tc::mbar_arrive_expect_tx(&zbar, (unsigned)(G * C * 4));
      for (int hl = 0; hl < G; ++hl) tc::bulk_load(zs + hl * C, z0 + hl * hstride, (unsigned)(C * 4), &zbar);
    }
    (void)tc::mbar_wait(&zbar, 0);
  }
  const uint32_t kneg = order_key(-INFINITY);
  // thread t owns chunks t + 512 m (m < MAXM, C <= 512 MAXM); packed keys stay in registers
  const int nm = (C + DK_THREADS - 1) / DK_THREADS;
  unsigned long long pk[MAXM];
#pragma unroll
  for (int m = 0; m < MAXM; ++m) {
    pk[m] = 0ull;
    const int c = tid + DK_THREADS * m;
    if (m < nm && c < C) {
      float zz;
      if (ZS) {
        zz = zs[c];
        for (int hl = 1; hl < G; ++hl) zz = fmaxf(zz, zs[hl * C + c]);
      } else {
        zz = z0[c];
        for (int hl = 1; hl < G; ++hl) zz = fmaxf(zz, z0[hl * hstride + c]);
      }
      const uint32_t key = order_key(zz);
      keys[c] = key;
      if (key > kneg) pk[m] = ((unsigned long long)key << 32) | (0xffffffffu - (uint32_t)c);
    }
  }
  RDL_TRACE_POINT(2, 2);
  // per-warp q-th largest packed key (0 when the warp has fewer than q valid keys)
  constexpr int NW = DK_THREADS / 32;
  const int qk = (K + NW - 1) / NW;
  {
    unsigned long long last = ~0ull, bound = 0ull;
    for (int r = 0; r < qk; ++r) {
      unsigned long long best = 0ull;
#pragma unroll
      for (int m = 0; m < MAXM; ++m)
        if (pk[m] < last && pk[m] > best) best = pk[m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const unsigned long long x = __shfl_xor_sync(0xffffffffu, best, o);
        best = x > best ? x : best;
      }
      last = best;
      bound = best;
      if (best == 0ull) break;
    }
    if (lane == 0) wbound[warp] = bound;
  }
  if (tid == 0) ncand_s = 0;
  __syncthreads();
  unsigned long long L0 = wbound[0];
#pragma unroll
  for (int w8 = 1; w8 < NW; ++w8) L0 = wbound[w8] < L0 ? wbound[w8] : L0;
  if (L0 == 0ull) L0 = 1ull;      // fewer than K valid keys in some warp: every valid key is a candidate
  // candidates: keys >= L0
#pragma unroll
  for (int m = 0; m < MAXM; ++m) {
    if (pk[m] >= L0) {
      const int slot = atomicAdd(&ncand_s, 1);
      if (slot < DK_MAXCAND) cand[slot] = pk[m];
    }
  }
  __syncthreads();
  const int ncand = ncand_s;
  int nsel;
  if (ncand <= DK_MAXCAND) {
    // exact rank of each candidate (keys are distinct)
    if (tid < ncand) {
      const unsigned long long mine = cand[tid];
      int rank = 0;
      for (int e = 0; e < ncand; ++e) rank += cand[e] > mine;
      if (rank < K) sel_s[rank] = (int)(0xffffffffu - (uint32_t)(mine & 0xffffffffull));
    }
    nsel = min(ncand, K);
    __syncthreads();
    // ascending chunk order
    int c_mine = 0, pos = 0;
    if (tid < nsel) {
      c_mine = sel_s[tid];
      for (int e = 0; e < nsel; ++e) pos += sel_s[e] < c_mine;
    }
    __syncthreads();
    if (tid < nsel) sel_s[pos] = c_mine;
    __syncthreads();
  } else {
    // heavy ties: the radix select over all keys (written for 256 threads; the other
    // threads take part in its barriers only)
    __syncthreads();
    nsel = cta_select_topk_t<DK_THREADS>(keys, C, K, hist, whist, warp_sums, bc, sel_s);
  }
  RDL_TRACE_POINT(2, 3);
  for (int e = tid; e < K * G; e += DK_THREADS) {
    const int k = e % K, hl = e / K;
    const int c = k < nsel ? sel_s[k] : -1;
    if (hl == 0) irow[k] = c;
    float z = -INFINITY;
    if (c >= 0) z = ZS ? zs[hl * C + c] : z0[hl * hstride + c];
    z_sel[((size_t)(b * Hq + g * G + hl) * Lq + i) * K + k] = z;
  }
  RDL_TRACE_POINT(2, 4);
}

// =====================================================================================
// dec_attn_kernel: chunk-major two-level attention for decode blocks.
//
// Work items: for KV group (b, g), every selected chunk c, with one task per row that
// selected it (second-level softmax over its 63 content keys); the local window is
// computed by dec_swa_kernel<true> while the top-K still runs.  The R CTAs of a group all
// build the same histogram of tasks per chunk from idx and split the prefix of (row pairs
// + one slab load) into R equal shares, so a chunk that every row selected costs one CTA
// as much as many sparse ones.  A CTA streams its chunks' K/V once through a TMA ring;
// each consumer warp computes two tasks of a slab at once (M = 16 = two rows x 8 head
// slots) with the probabilities kept in registers (no shared-memory round trip), and
// writes o_part[b,i,g,k] = the softmax-normalised output of chunk idx[k].
// dec_comb_kernel merges a row's window part and chunk outputs in a fixed order.
// =====================================================================================
constexpr int AT_CONS = 15;
constexpr int AT_THREADS = (AT_CONS + 1) * 32;
constexpr int AT_STAGE_BYTES = 32768;
constexpr int AT_MAXC = 2048;            // chunks per sequence on this path
constexpr int AT_QROWS = 32;             // query rows per sequence on this path
constexpr int AT_SLAB_WORK = 2;          // partition weight of one slab load, in row pairs

// window slabs a row at position p touches: [wlo(p), whi(p)] (w >= 0)
__device__ __forceinline__ int win_lo(int p, int w) { return max(0, p - w) / S; }
__device__ __forceinline__ int win_hi(int p, int w, int L) { return min(L - 1, p + w) / S; }
// most window slabs of one row: 2w+1 keys span at most 2w/64 + 2 slabs
__host__ __device__ inline int max_win_slabs(int w) { return w < 0 ? 0 : (2 * w) / S + 2; }

struct AttnSmem {
  int ring, qs, idx, pos, hist, pre, list, bar, misc, total;
};
__host__ __device__ inline AttnSmem attn_smem(int stages, int Lq, int K, int C) {
  AttnSmem s{};
  int off = 0;
  s.ring = off; off += stages * AT_STAGE_BYTES;
  s.qs = off;   off += Lq * 2048;
  s.idx = off;  off += ((Lq * K + 3) & ~3) * 4;
  s.pos = off;  off += ((Lq + 3) & ~3) * 4;
  s.hist = off; off += ((C + 3) & ~3) * 4;
  s.pre = off;  off += ((C + 3) & ~3) * 4;
  s.list = off; off += ((Lq * K + 3) & ~3) * 4;
  s.bar = off;  off += 16 * stages;
  s.misc = off; off += 256;
  s.total = off + 1024;
  return s;
}

// byte offset of (row, col) in a K/V slab tile ([2 halves][64 rows][128 B], 128-byte swizzle)
__device__ __forceinline__ uint32_t kv_off(int row, int col) {
  return (uint32_t)((col >> 6) * 8192 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2);
}

// Exclusive scan of one int per thread over the whole CTA (blockDim.x <= 1024); returns the
// thread's exclusive prefix and the CTA total.  ws: blockDim.x / 32 ints of shared memory.
__device__ __forceinline__ int cta_excl_scan(int v, int* ws, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) ws[warp] = x;
  __syncthreads();
  int basev = 0, tot = 0;
  for (int w8 = 0; w8 < nw; ++w8) {
    const int t = ws[w8];
    if (w8 < warp) basev += t;
    tot += t;
  }
  __syncthreads();
  total = tot;
  return basev + x - v;
}

// Exclusive scan of two ints per thread over the whole CTA (blockDim.x <= 1024); returns the
// thread's two exclusive prefixes and the two CTA totals.  ws: 2 * blockDim.x / 32 ints.
__device__ __forceinline__ int2 cta_excl_scan2(int a, int bv, int* ws, int& ta, int& tb) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  int x = a, y = bv;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int xa = __shfl_up_sync(0xffffffffu, x, o), ya = __shfl_up_sync(0xffffffffu, y, o);
    if (lane >= o) {
      x += xa;
      y += ya;
    }
  }
  if (lane == 31) {
    ws[2 * warp] = x;
    ws[2 * warp + 1] = y;
  }
  __syncthreads();
  int ba = 0, bb = 0, sa = 0, sb = 0;
  for (int w8 = 0; w8 < nw; ++w8) {
    const int va = ws[2 * w8], vb = ws[2 * w8 + 1];
    if (w8 < warp) {
      ba += va;
      bb += vb;
    }
    sa += va;
    sb += vb;
  }
  __syncthreads();
  ta = sa;
  tb = sb;
  return make_int2(ba + x - a, bb + y - bv);
}

// task word: row << 8 | slot (slot < 128)

template <bool ROUTE>
__global__ void __launch_bounds__(AT_THREADS, 1)
    dec_attn_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                    const __nv_bfloat16* __restrict__ kv_base_k, const __nv_bfloat16* __restrict__ kv_base_v,
                    const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ q_pos,
                    const int32_t* __restrict__ idx, int L, int Lq, int Hq, int Hkv, int K, int w, int flags,
                    int R, int stages, float sl2, float* __restrict__ o_part) {
  constexpr int D = 128;
  extern __shared__ unsigned char at_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(at_raw) + 1023) & ~uintptr_t(1023));
  const int C = L / S, G = Hq / Hkv;
  const int Kt = ROUTE ? K : 0;
  const AttnSmem SL = attn_smem(stages, Lq, Kt, C);
  unsigned char* ring = base + SL.ring;
  unsigned char* qs = base + SL.qs;
  int* idx_s = reinterpret_cast<int*>(base + SL.idx);
  int* pos_s = reinterpret_cast<int*>(base + SL.pos);
  int* hist = reinterpret_cast<int*>(base + SL.hist);
  int* pre = reinterpret_cast<int*>(base + SL.pre);
  int* list = reinterpret_cast<int*>(base + SL.list);
  uint64_t* full = reinterpret_cast<uint64_t*>(base + SL.bar);
  uint64_t* empty = full + stages;
  int* misc = reinterpret_cast<int*>(base + SL.misc);   // [0] c_lo [1] c_hi [2] abort [3..4] scan
  RDL_TRACE_POINT(3, 0);

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int item = blockIdx.x, j = item % R, g = (item / R) % Hkv, b = item / (R * Hkv);
  const size_t kvrow0 = (size_t)(b * Hkv + g) * L;

  if (tid == 0) {
    for (int st = 0; st < stages; ++st) {
      tc::mbar_init(&full[st], 1);
      tc::mbar_init(&empty[st], AT_CONS);
    }
    tc::mbar_fence_init();
    misc[0] = INT_MAX;
    misc[1] = -1;
    misc[2] = 0;
  }
  // ---------------- prologue: inputs of the call only (this kernel starts early only when
  // every kernel before the call has completed): positions and the query rows (waited for
  // with the idx rows)
  for (int e = tid; e < Lq; e += AT_THREADS) pos_s[e] = q_pos ? __ldcg(q_pos + (size_t)b * Lq + e) : e;
  for (int e = tid; e < Lq * 8 * 16 && tid < AT_CONS * 32; e += AT_CONS * 32) {   // consumer threads only
    const int i = e >> 7, hd = (e >> 4) & 7, u = e & 15;
    unsigned char* dst = qs + i * 2048 + hd * 256 + ((u ^ hd) << 4);
    if (hd < G)
      cp_async16(smem_u32(dst), q + ((size_t)(b * Lq + i) * Hq + g * G + hd) * D + u * 8);
    else
      *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
  }
  cp_async_commit();                      // group 1: query rows
  for (int c = tid; c < C; c += AT_THREADS) hist[c] = 0;
  grid_dep_wait();
  grid_dep_launch();
  RDL_TRACE_POINT(3, 1);

  // ---------------- idx rows of the group
  const int nent = Lq * Kt;
  const int32_t* ib = ROUTE ? idx + (size_t)(b * Hkv + g) * Lq * K : nullptr;
  if (ROUTE) {
    if ((nent & 3) == 0) {
      for (int e = tid; e < nent / 4; e += AT_THREADS) cp_async16(smem_u32(idx_s + 4 * e), ib + 4 * e);
    } else {
      for (int e = tid; e < nent; e += AT_THREADS) idx_s[e] = ib[e];
    }
  }
  cp_async_commit();                      // group 2: idx
  cp_async_wait<0>();
  __syncthreads();
  RDL_TRACE_POINT(3, 4);
  // ---------------- chunk tasks per slab (the same on every CTA of the group)
  auto chunk_ok = [&](int e, int c) -> bool {   // entry e of idx_s holds chunk c >= 0
    if (c >= C) return false;
    if (flags & RDL_FLAG_CHECKS) return chunk_eligible(c, pos_s[e / K], w);
    return true;
  };
  if (ROUTE) {
    for (int e = tid; e < nent; e += AT_THREADS) {
      const int c = idx_s[e];
      if (c < 0) continue;
      if (!chunk_ok(e, c)) {
        if (flags & RDL_FLAG_CHECKS) record_status(RDL_ERR_DEVICE_CHECK);
        continue;
      }
      atomicAdd(&hist[c], 1);
    }
  }
  __syncthreads();
  // One scan gives both prefixes in chunk order: pre[c] = first list position of slab c's
  // tasks, and the work prefix, work of slab c = its row pairs plus one slab load (weighted
  // AT_SLAB_WORK pairs).  Slab c belongs to CTA floor((work prefix(c) + work(c) / 2) * R /
  // total work), the share that holds the slab's midpoint: contiguous slab ranges of equal
  // work, a heavy slab overshooting a share by at most half its work.
  int* scan_ws = misc + 32;                                  // 32 ints
  {
    const int seg = (C + AT_THREADS - 1) / AT_THREADS;
    const int s0 = min(C, tid * seg), s1 = min(C, s0 + seg);
    int lt = 0, lw = 0;
    for (int c = s0; c < s1; ++c) {
      const int n = hist[c];
      lt += n;
      lw += n > 0 ? (n + 1) / 2 + AT_SLAB_WORK : 0;
    }
    int tot_t, tot_w;
    const int2 pr = cta_excl_scan2(lt, lw, scan_ws, tot_t, tot_w);
    int rt = pr.x, rw = pr.y;
    // rw * R < 2^31: at most C slabs x (Lq/2 + K + AT_SLAB_WORK) units x 148 CTAs
    for (int c = s0; c < s1; ++c) {
      const int n = hist[c];
      pre[c] = rt;
      rt += n;
      if (n > 0) {
        const int wc = (n + 1) / 2 + AT_SLAB_WORK;
        const int owner = min(R - 1, ((rw + wc / 2) * R) / tot_w);   // share holding the slab's midpoint
        if (owner == j) {
          atomicMin(&misc[0], c);
          atomicMax(&misc[1], c);
        }
        rw += wc;
      }
    }
  }
  RDL_TRACE_POINT(3, 6);
  __syncthreads();
  const int c_lo = misc[0], c_hi = misc[1] + 1;     // empty when c_lo > c_hi - 1

  if (warp == AT_CONS) {
    // ---------------- TMA producer: starts while the consumers build the task lists
    if (lane == 0) {
      int u = 0;
      int last_issued[4] = {-1, -1, -1, -1};
      for (int c = c_lo; c < c_hi; ++c) {
        if (hist[c] == 0) continue;
        const int st = u % stages, n = u / stages;
        if (n > 0 && !tc::mbar_wait(&empty[st], (unsigned)(n - 1) & 1u)) {
          misc[2] = 1;
          break;
        }
        if (misc[2]) break;
        unsigned char* dst = ring + st * AT_STAGE_BYTES;
        tc::mbar_arrive_expect_tx(&full[st], AT_STAGE_BYTES);
        tc::tma_load_3d(dst, &kmap, 0, (int)(kvrow0 + (size_t)S * c), 0, &full[st]);
        tc::tma_load_3d(dst + 16384, &vmap, 0, (int)(kvrow0 + (size_t)S * c), 0, &full[st]);
        last_issued[st] = u;
        ++u;
      }
      for (int st = 0; st < stages; ++st)
        if (last_issued[st] >= 0) (void)tc::mbar_wait(&full[st], (unsigned)(last_issued[st] / stages) & 1u);
    }
    __syncwarp();
    __syncthreads();
    return;
  }

  // ---------------- consumer warps only from here (named barrier 1, AT_CONS warps)
  const int lbase = c_lo < c_hi ? pre[c_lo] : 0;   // list positions relative to this CTA
  const int lcap = Lq * Kt;
  asm volatile("bar.sync 1, %0;\n" ::"n"(AT_CONS * 32) : "memory");
  if (ROUTE && c_lo < c_hi) {
    for (int e = tid; e < nent; e += AT_CONS * 32) {
      const int c = idx_s[e];
      if (c < c_lo || c >= c_hi || !chunk_ok(e, c)) continue;
      const int slot = atomicAdd(&pre[c], 1) - lbase;
      if (slot < lcap) list[slot] = ((e / K) << 8) | (e % K);
      else record_status(RDL_ERR_DEVICE_CHECK);
    }
  }
  RDL_TRACE_POINT(3, 2);
  // after the scatter pre[c] = end of slab c's tasks (absolute); start = end - hist[c]

  // ---------------- consumer warps: pairs of tasks, pair index % AT_CONS == warp
  cp_async_wait<0>();
  asm volatile("bar.sync 1, %0;\n" ::"n"(AT_CONS * 32) : "memory");   // query rows visible to every consumer
  int u = 0, pair0 = 0;
  for (int c = c_lo; c < c_hi; ++c) {
    const int n = hist[c];
    if (n == 0) continue;
    const int st = u % stages;
    if (!tc::mbar_wait(&full[st], (unsigned)(u / stages) & 1u)) {
      misc[2] = 1;
      break;
    }
    if (u == 0) RDL_TRACE_POINT(3, 3);
    const uint32_t kst = smem_u32(ring + st * AT_STAGE_BYTES), vst = kst + 16384;
    const int tbeg = pre[c] - n - lbase, npair = (n + 1) / 2;
    int pfirst = (warp - pair0 % AT_CONS + AT_CONS) % AT_CONS;
    for (int pp = pfirst; pp < npair; pp += AT_CONS) {
      const int tA = list[tbeg + 2 * pp];
      const bool hasB = 2 * pp + 1 < n;
      const int tB = hasB ? list[tbeg + 2 * pp + 1] : tA;
      const int iA = tA >> 8, iB = tB >> 8;
      // ---- S = Q K^T for rows (iA heads 0-7, iB heads 0-7) x 64 keys
      float sc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
      {
        const int mi = lane >> 3;
        const uint32_t qrow = smem_u32(qs + ((mi & 1) ? iB : iA) * 2048) + (lane & 7) * 256;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          uint32_t a[4];
          const int uq = 2 * ks + (mi >> 1);
          ldsm_x4(qrow + ((uq ^ (lane & 7)) << 4), a[0], a[1], a[2], a[3]);
#pragma unroll
          for (int np = 0; np < 4; ++np) {
            uint32_t b0, b1, b2, b3;
            const int key = 16 * np + 8 * (mi >> 1) + (lane & 7), col = 16 * ks + 8 * (mi & 1);
            ldsm_x4(kst + kv_off(key, col), b0, b1, b2, b3);
            mma_bf16(sc[2 * np], a, b0, b1);
            mma_bf16(sc[2 * np + 1], a, b2, b3);
          }
        }
      }
      // ---- softmax over the chunk's content keys (row gq: task A, row gq + 8: task B)
      float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = 8 * nt + 2 * tq + (e & 1);
          const int hb = e >> 1;
          const float v = key < CONTENT ? sc[nt][e] * sl2 : -INFINITY;
          sc[nt][e] = v;
          mx[hb] = fmaxf(mx[hb], v);
        }
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        mx[hb] = fmaxf(mx[hb], __shfl_xor_sync(0xffffffffu, mx[hb], 1));
        mx[hb] = fmaxf(mx[hb], __shfl_xor_sync(0xffffffffu, mx[hb], 2));
      }
      float sm[2] = {0.f, 0.f};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int hb = e >> 1;
          const float pv = fast_exp2(sc[nt][e] - mx[hb]);   // masked: exp2(-inf) = 0
          sc[nt][e] = pv;
          sm[hb] += pv;
        }
#pragma unroll
      for (int hb = 0; hb < 2; ++hb) {
        sm[hb] += __shfl_xor_sync(0xffffffffu, sm[hb], 1);
        sm[hb] += __shfl_xor_sync(0xffffffffu, sm[hb], 2);
      }
      const float fA = 1.f / sm[0], fB = 1.f / sm[1];
      // P as bf16 A fragments (FA2 layout: the S accumulators of n-tiles 2kk, 2kk+1)
      uint32_t pa[4][4];
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        pa[kk][0] = pack_bf16(sc[2 * kk][0] * fA, sc[2 * kk][1] * fA);
        pa[kk][1] = pack_bf16(sc[2 * kk][2] * fB, sc[2 * kk][3] * fB);
        pa[kk][2] = pack_bf16(sc[2 * kk + 1][0] * fA, sc[2 * kk + 1][1] * fA);
        pa[kk][3] = pack_bf16(sc[2 * kk + 1][2] * fB, sc[2 * kk + 1][3] * fB);
      }
      float* dstA = nullptr;
      float* dstB = nullptr;
      {
        const int slotA = tA & 127, slotB = tB & 127;
        const size_t rgA = (size_t)(b * Lq + iA) * Hkv + g, rgB = (size_t)(b * Lq + iB) * Hkv + g;
        if (gq < G) {
          dstA = o_part + ((rgA * K + slotA) * G + gq) * D;
          if (hasB) dstB = o_part + ((rgB * K + slotB) * G + gq) * D;
        }
      }
      // ---- O = P V, 64 dims at a time
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float oc[8][4];
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) oc[nt][0] = oc[nt][1] = oc[nt][2] = oc[nt][3] = 0.f;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const int mi = lane >> 3;
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            uint32_t b0, b1, b2, b3;
            const int key = 16 * kk + 8 * (mi & 1) + (lane & 7), col = 64 * half + 16 * m + 8 * (mi >> 1);
            ldsm_x4_t(vst + kv_off(key, col), b0, b1, b2, b3);
            mma_bf16(oc[2 * m], pa[kk], b0, b1);
            mma_bf16(oc[2 * m + 1], pa[kk], b2, b3);
          }
        }
        if (dstA) {
#pragma unroll
          for (int nt = 0; nt < 8; ++nt)
            *reinterpret_cast<float2*>(dstA + 64 * half + 8 * nt + 2 * tq) = make_float2(oc[nt][0], oc[nt][1]);
        }
        if (dstB) {
#pragma unroll
          for (int nt = 0; nt < 8; ++nt)
            *reinterpret_cast<float2*>(dstB + 64 * half + 8 * nt + 2 * tq) = make_float2(oc[nt][2], oc[nt][3]);
        }
      }
    }
    if (u == 0) RDL_TRACE_POINT(3, 7);
    pair0 += npair;
    __syncwarp();
    if (lane == 0) tc::mbar_arrive(&empty[st]);
    ++u;
  }
  __syncthreads();   // pairs with the producer's final barrier
  RDL_TRACE_POINT(3, 5);
}

// =====================================================================================
// dec_swa_kernel: bidirectional sliding window for decode blocks, one launch.
// CTA = (b, g, pair of query rows); warp w streams window slabs w, w + SW_WARPS, ... of the
// pair through its own shared-memory slot (TMA), keeps an online softmax per row (M = 16 =
// two rows x 8 head slots), and the warps' partial states are merged in a fixed order.
// ROUTE_WIN: the local-window part of a route layer.  It reads only inputs of the call, so
// it runs while the top-K of the same step is still running: it releases its dependent at
// once and waits for its own predecessor only before its first global store (its completion
// then implies the predecessor's, and no store overtakes a read of the predecessor).  It
// writes the window's (max, sum) and unnormalised vector per (row, head) for
// dec_comb_kernel instead of the normalised output.
// =====================================================================================
constexpr int SW_WARPS = 6;

__host__ __device__ inline int swa_smem() { return 1024 + SW_WARPS * AT_STAGE_BYTES + 2 * 2048 + 64 * SW_WARPS; }

template <bool ROUTE_WIN>
__global__ void __launch_bounds__(SW_WARPS * 32, 1)
    dec_swa_kernel(const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
                   const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ q_pos, int L, int Lq, int Hq,
                   int Hkv, int w, float sl2, __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
                   float* __restrict__ ow, float2* __restrict__ ml) {
  constexpr int D = 128;
  extern __shared__ unsigned char sw_raw[];
  unsigned char* base = reinterpret_cast<unsigned char*>((reinterpret_cast<uintptr_t>(sw_raw) + 1023) & ~uintptr_t(1023));
  unsigned char* slabs = base;                                   // [SW_WARPS][32 KB]
  unsigned char* qs = slabs + SW_WARPS * AT_STAGE_BYTES;         // [2 rows][8 heads][256 B]
  uint64_t* bar = reinterpret_cast<uint64_t*>(qs + 2 * 2048);    // one per warp
  const int C = L / S, G = Hq / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  const int npair = (Lq + 1) / 2;
  const int pr = blockIdx.x % npair, g = (blockIdx.x / npair) % Hkv, b = blockIdx.x / (npair * Hkv);
  const int iA = 2 * pr, iB = min(2 * pr + 1, Lq - 1);
  const bool hasB = 2 * pr + 1 < Lq;
  if (tid == 0) {
    for (int x = 0; x < SW_WARPS; ++x) tc::mbar_init(&bar[x], 1);
    tc::mbar_fence_init();
  }
  if (!ROUTE_WIN) grid_dep_wait();
  grid_dep_launch();
  RDL_TRACE_POINT(5, 0);
  const int pA = q_pos ? q_pos[(size_t)b * Lq + iA] : iA;
  const int pB = q_pos ? q_pos[(size_t)b * Lq + iB] : iB;
  // query rows of the pair: [row][8 heads][256 B], 16-byte units ^ head; head 7+ zero
  for (int e = tid; e < 2 * 8 * 16; e += SW_WARPS * 32) {
    const int r = e >> 7, hd = (e >> 4) & 7, u = e & 15;
    unsigned char* dst = qs + r * 2048 + hd * 256 + ((u ^ hd) << 4);
    if (hd < G)
      cp_async16(smem_u32(dst), q + ((size_t)(b * Lq + (r ? iB : iA)) * Hq + g * G + hd) * D + u * 8);
    else
      *reinterpret_cast<uint4*>(dst) = make_uint4(0u, 0u, 0u, 0u);
  }
  cp_async_commit();
  // slabs of the two windows: [loA, hiA] and [loB, hiB] (the union, in order)
  int loA = win_lo(pA, w), hiA = win_hi(pA, w, L), loB = win_lo(pB, w), hiB = win_hi(pB, w, L);
  if (loB < loA) {
    const int t0 = loA, t1 = hiA;
    loA = loB; hiA = hiB; loB = t0; hiB = t1;
  }
  const int nA = max(0, hiA - loA + 1);
  const int startB = max(loB, hiA + 1), nB = max(0, hiB - startB + 1);
  const int nsl = nA + nB;
  auto slab_at = [&](int u) { return u < nA ? loA + u : startB + (u - nA); };
  // this warp's first slab
  unsigned char* my = slabs + warp * AT_STAGE_BYTES;
  const size_t kvrow0 = (size_t)(b * Hkv + g) * L;
  int phase = 0;
  if (lane == 0 && warp < nsl) {
    const int t = slab_at(warp);
    tc::mbar_arrive_expect_tx(&bar[warp], AT_STAGE_BYTES);
    tc::tma_load_3d(my, &kmap, 0, (int)(kvrow0 + (size_t)S * t), 0, &bar[warp]);
    tc::tma_load_3d(my + 16384, &vmap, 0, (int)(kvrow0 + (size_t)S * t), 0, &bar[warp]);
  }
  cp_async_wait<0>();
  __syncthreads();
  // A fragments of the pair's query rows, all 8 k-steps
  uint32_t qa[8][4];
  {
    const int mi = lane >> 3;
    const uint32_t qrow = smem_u32(qs + (mi & 1) * 2048) + (lane & 7) * 256;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const int uq = 2 * ks + (mi >> 1);
      ldsm_x4(qrow + ((uq ^ (lane & 7)) << 4), qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
    }
  }
  float mrun[2] = {-INFINITY, -INFINITY}, lrun[2] = {0.f, 0.f};
  float oc[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) oc[nt][0] = oc[nt][1] = oc[nt][2] = oc[nt][3] = 0.f;
  for (int u = warp; u < nsl; u += SW_WARPS) {
    const int t = slab_at(u);
    if (!tc::mbar_wait(&bar[warp], (unsigned)phase)) break;
    phase ^= 1;
    const uint32_t kst = smem_u32(my), vst = kst + 16384;
    float sc[8][4];
#pragma unroll
    for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
    {
      const int mi = lane >> 3;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
#pragma unroll
        for (int np = 0; np < 4; ++np) {
          uint32_t b0, b1, b2, b3;
          const int key = 16 * np + 8 * (mi >> 1) + (lane & 7), col = 16 * ks + 8 * (mi & 1);
          ldsm_x4(kst + kv_off(key, col), b0, b1, b2, b3);
          mma_bf16(sc[2 * np], qa[ks], b0, b1);
          mma_bf16(sc[2 * np + 1], qa[ks], b2, b3);
        }
    }
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hb = e >> 1, p = hb ? pB : pA;
        const int j = S * t + 8 * nt + 2 * tq + (e & 1);
        const bool in = (hb == 0 || hasB) && j >= p - w && j <= p + w;
        const float v = in ? sc[nt][e] * sl2 : -INFINITY;
        sc[nt][e] = v;
        mx[hb] = fmaxf(mx[hb], v);
      }
    float alpha[2], mnew[2];
#pragma unroll
    for (int hb = 0; hb < 2; ++hb) {
      mx[hb] = fmaxf(mx[hb], __shfl_xor_sync(0xffffffffu, mx[hb], 1));
      mx[hb] = fmaxf(mx[hb], __shfl_xor_sync(0xffffffffu, mx[hb], 2));
      mnew[hb] = fmaxf(mrun[hb], mx[hb]);
      alpha[hb] = mnew[hb] == -INFINITY ? 1.f : fast_exp2(mrun[hb] - mnew[hb]);
    }
    float sm[2] = {0.f, 0.f};
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hb = e >> 1;
        const float pv = mnew[hb] == -INFINITY ? 0.f : fast_exp2(sc[nt][e] - mnew[hb]);
        sc[nt][e] = pv;
        sm[hb] += pv;
      }
#pragma unroll
    for (int hb = 0; hb < 2; ++hb) {
      sm[hb] += __shfl_xor_sync(0xffffffffu, sm[hb], 1);
      sm[hb] += __shfl_xor_sync(0xffffffffu, sm[hb], 2);
      lrun[hb] = lrun[hb] * alpha[hb] + sm[hb];
      mrun[hb] = mnew[hb];
    }
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      oc[nt][0] *= alpha[0];
      oc[nt][1] *= alpha[0];
      oc[nt][2] *= alpha[1];
      oc[nt][3] *= alpha[1];
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      a[0] = pack_bf16(sc[2 * kk][0], sc[2 * kk][1]);
      a[1] = pack_bf16(sc[2 * kk][2], sc[2 * kk][3]);
      a[2] = pack_bf16(sc[2 * kk + 1][0], sc[2 * kk + 1][1]);
      a[3] = pack_bf16(sc[2 * kk + 1][2], sc[2 * kk + 1][3]);
      const int mi = lane >> 3;
#pragma unroll
      for (int m = 0; m < 8; ++m) {
        uint32_t b0, b1, b2, b3;
        const int key = 16 * kk + 8 * (mi & 1) + (lane & 7), col = 16 * m + 8 * (mi >> 1);
        ldsm_x4_t(vst + kv_off(key, col), b0, b1, b2, b3);
        mma_bf16(oc[2 * m], a, b0, b1);
        mma_bf16(oc[2 * m + 1], a, b2, b3);
      }
    }
    __syncwarp();
    // next slab of this warp into the same slot
    const int un = u + SW_WARPS;
    if (lane == 0 && un < nsl) {
      const int tn = slab_at(un);
      tc::fence_proxy_async();
      tc::mbar_arrive_expect_tx(&bar[warp], AT_STAGE_BYTES);
      tc::tma_load_3d(my, &kmap, 0, (int)(kvrow0 + (size_t)S * tn), 0, &bar[warp]);
      tc::tma_load_3d(my + 16384, &vmap, 0, (int)(kvrow0 + (size_t)S * tn), 0, &bar[warp]);
    }
  }
  // ---- fixed-order merge of the warps' states through shared memory (slabs are idle now)
  __syncthreads();
  float* part = reinterpret_cast<float*>(slabs) + warp * (16 * 128 + 64);   // [16 rows][128] + m, l
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) {
    part[gq * 128 + 8 * nt + 2 * tq] = oc[nt][0];
    part[gq * 128 + 8 * nt + 2 * tq + 1] = oc[nt][1];
    part[(gq + 8) * 128 + 8 * nt + 2 * tq] = oc[nt][2];
    part[(gq + 8) * 128 + 8 * nt + 2 * tq + 1] = oc[nt][3];
  }
  if (tq == 0) {
    part[2048 + gq] = mrun[0];
    part[2048 + 8 + gq] = mrun[1];
    part[2048 + 16 + gq] = lrun[0];
    part[2048 + 24 + gq] = lrun[1];
  }
  __syncthreads();
  // thread: (row of 16, 4 dims) cells e = tid + 192 u; rows 0-7 = row A heads, 8-15 = row B.
  // The merged cells are kept in registers and stored after the wait below.
  constexpr int NCELL = (16 * 32 + SW_WARPS * 32 - 1) / (SW_WARPS * 32);
  const float* p0 = reinterpret_cast<const float*>(slabs);
  float cM[NCELL], cL[NCELL], cacc[NCELL][4];
#pragma unroll
  for (int u = 0; u < NCELL; ++u) {
    const int e = tid + SW_WARPS * 32 * u;
    const int row = (e >> 5) & 15, d4 = (e & 31) * 4, hd = row & 7, hb = row >> 3;
    float M = -INFINITY;
    for (int x = 0; x < SW_WARPS; ++x) M = fmaxf(M, p0[x * (2048 + 64) + 2048 + hb * 8 + hd]);
    float Lsum = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int x = 0; x < SW_WARPS; ++x) {
      const float* px = p0 + x * (2048 + 64);
      const float mxx = px[2048 + hb * 8 + hd];
      if (mxx == -INFINITY) continue;
      const float f = fast_exp2(mxx - M);
      Lsum += f * px[2048 + 16 + hb * 8 + hd];
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[c] += f * px[row * 128 + d4 + c];
    }
    cM[u] = M;
    cL[u] = Lsum;
#pragma unroll
    for (int c = 0; c < 4; ++c) cacc[u][c] = acc[c];
  }
  // ROUTE_WIN: the window part goes to a workspace the previous kernel on the stream may
  // still be reading (the combine of an earlier call on the same workspace), so the stores
  // wait for the predecessor; everything above touched inputs and shared memory only.
  if (ROUTE_WIN) grid_dep_wait();
#pragma unroll
  for (int u = 0; u < NCELL; ++u) {
    const int e = tid + SW_WARPS * 32 * u;
    const int row = (e >> 5) & 15, d4 = (e & 31) * 4, hd = row & 7, hb = row >> 3;
    if (e >= 16 * 32 || hd >= G || (hb == 1 && !hasB)) continue;
    const float M = cM[u], Lsum = cL[u];
    const int i = hb ? iB : iA, h = g * G + hd;
    if (ROUTE_WIN) {
      // (max in natural-log units, sum) and the vector relative to that max
      const size_t rh = (size_t)(b * Lq + i) * Hq + h;
      *reinterpret_cast<float4*>(ow + rh * D + d4) = make_float4(cacc[u][0], cacc[u][1], cacc[u][2], cacc[u][3]);
      if (d4 == 0) ml[rh] = make_float2(Lsum > 0.f ? M * LN2 : -INFINITY, Lsum);
      continue;
    }
    const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
    __nv_bfloat16* orow = o + ((size_t)(b * Lq + i) * Hq + h) * D + d4;
    const __nv_bfloat162 o01 = __floats2bfloat162_rn(cacc[u][0] * inv, cacc[u][1] * inv);
    const __nv_bfloat162 o23 = __floats2bfloat162_rn(cacc[u][2] * inv, cacc[u][3] * inv);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t*>(&o01);
    pk.y = *reinterpret_cast<const uint32_t*>(&o23);
    *reinterpret_cast<uint2*>(orow) = pk;
    if (lse && d4 == 0) lse[(size_t)(b * Hq + h) * Lq + i] = Lsum > 0.f ? (M + log2f(Lsum)) * LN2 : -INFINITY;
  }
  RDL_TRACE_POINT(5, 1);
  (void)C;
}

// =====================================================================================
// dec_comb_kernel: one warp per (b, i, h); lane l owns dims 4l .. 4l+3.  Merges the
// window part (max, sum, unnormalised vector) and, on route layers, the chunk outputs with
// weights e^{z_c}: one partition, o = sum(weight * vector) / sum(weight), in a fixed order.
// Chunk outputs are loaded in batches before their weights are known (unused loads are
// harmless).
// =====================================================================================
constexpr int COMB_SPREAD_SMEM = 120 * 1024;   // dynamic shared memory requested (unused)
template <bool ROUTE>
__global__ void __launch_bounds__(256) dec_comb_kernel(const int32_t* __restrict__ q_pos,
                                                       const int32_t* __restrict__ idx,
                                                       const float* __restrict__ z_sel,
                                                       const float* __restrict__ o_part,
                                                       const float* __restrict__ ow,
                                                       const float2* __restrict__ ml, int B, int L, int Lq,
                                                       int Hq, int Hkv, int K, int w, int flags,
                                                       __nv_bfloat16* __restrict__ o, float* __restrict__ lse) {
  constexpr int D = 128;
  grid_dep_wait();
  grid_dep_launch();
  RDL_TRACE_POINT(4, 1);
  const int lane = threadIdx.x & 31;
  const long long item = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (item >= (long long)B * Lq * Hq) return;
  const int h = (int)(item % Hq);
  const int i = (int)((item / Hq) % Lq);
  const int b = (int)(item / ((long long)Hq * Lq));
  const int C = L / S, G = Hq / Hkv, g = h / G, hl = h % G;
  const int p = q_pos ? q_pos[(size_t)b * Lq + i] : i;
  if (ROUTE && is_mask_slot(p)) return;
  const size_t rh = (size_t)(b * Lq + i) * Hq + h;
  const size_t rg = (size_t)(b * Lq + i) * Hkv + g;
  // every load that does not depend on a weight is issued first: the window part (absent
  // when w < 0 or the window is empty: sum 0), the chunk ids and logits (lanes k, k+32 hold
  // slot k) and the first 16 chunk outputs
  float2 wml = make_float2(-INFINITY, 0.f);
  float4 vw = make_float4(0.f, 0.f, 0.f, 0.f);
  if (w >= 0) {
    wml = ml[rh];
    vw = *reinterpret_cast<const float4*>(ow + rh * D + 4 * lane);
  }
  int ck[2] = {-1, -1};
  float zr[2] = {-INFINITY, -INFINITY};
  const float* pbase = o_part + (rg * K * G + hl) * D + 4 * lane;
  float4 v0[16];
  if (ROUTE) {
    const int32_t* irow = idx + ((size_t)(b * Hkv + g) * Lq + i) * K;
    const float* zrow = z_sel + ((size_t)(b * Hq + h) * Lq + i) * K;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int k = lane + 32 * u;
      if (k < K) {
        ck[u] = irow[k];
        zr[u] = zrow[k];
      }
    }
#pragma unroll
    for (int u = 0; u < 16; ++u)
      v0[u] = u < K ? *reinterpret_cast<const float4*>(pbase + (size_t)u * G * D) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  float zk[2] = {-INFINITY, -INFINITY};
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    const int c = ck[u];
    bool ok = ROUTE && c >= 0 && c < C;
    if (ok && (flags & RDL_FLAG_CHECKS) && !chunk_eligible(c, p, w)) ok = false;
    if (ok) zk[u] = zr[u];
  }
  const bool has_w = wml.y > 0.f;
  float M = fmaxf(zk[0], zk[1]);
  M = warp_max(M);
  if (has_w) M = fmaxf(M, wml.x);
  if (M == -INFINITY) M = 0.f;
  const float ew = has_w ? expf(wml.x - M) : 0.f;           // window weight e^{m - M}
  const float ek0 = zk[0] == -INFINITY ? 0.f : expf(zk[0] - M);
  const float ek1 = zk[1] == -INFINITY ? 0.f : expf(zk[1] - M);
  const float Zs = ew * wml.y + warp_sum(ek0 + ek1);
  float4 acc = make_float4(ew * vw.x, ew * vw.y, ew * vw.z, ew * vw.w);
  if (ROUTE) {
    for (int k0 = 0; k0 < K; k0 += 16) {
      float4 v[16];
#pragma unroll
      for (int u = 0; u < 16; ++u)
        v[u] = k0 == 0 ? v0[u]
                       : (k0 + u < K ? *reinterpret_cast<const float4*>(pbase + (size_t)(k0 + u) * G * D)
                                     : make_float4(0.f, 0.f, 0.f, 0.f));
#pragma unroll
      for (int u = 0; u < 16; ++u) {
        const int k = k0 + u;
        const float f = __shfl_sync(0xffffffffu, (k < 32) ? ek0 : ek1, k & 31);
        if (k < K && f != 0.f) {
          acc.x += f * v[u].x; acc.y += f * v[u].y; acc.z += f * v[u].z; acc.w += f * v[u].w;
        }
      }
    }
  }
  const float inv = Zs > 0.f ? 1.f / Zs : 0.f;
  __nv_bfloat16* orow = o + ((size_t)(b * Lq + i) * Hq + h) * D + 4 * lane;
  const __nv_bfloat162 o01 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
  const __nv_bfloat162 o23 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
  uint2 pk;
  pk.x = *reinterpret_cast<const uint32_t*>(&o01);
  pk.y = *reinterpret_cast<const uint32_t*>(&o23);
  *reinterpret_cast<uint2*>(orow) = pk;
  if (lse && lane == 0) lse[(size_t)(b * Hq + h) * Lq + i] = Zs > 0.f ? M + logf(Zs) : -INFINITY;
}

}  // namespace dec
}  // namespace rdl
