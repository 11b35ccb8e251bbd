// Route score on tensor cores (bf16 inputs, d = 128), the prefill-sized path.
//
// The score of query row i, head h, chunk c is (Figure 3 caption of Prefilling-dLLM v2:
// a content query adds a low-rank residual and scores the summaries; the pooling entropy
// is the second signal)
//     z = tau * (q_h + u_h) . s_c,h - lambda * H_c,h ,   u = (x W_down) W_up,
// and because (t W_up)_h . s = t . (W_up,h s) with t = x W_down, it is computed as
//     z = tau * (q_h . s + t . s'_c,h) - lambda * H,      s'_c,h = W_up,h s_c,h  (rank r)
// so the residual-adapted query q_res is never materialised.
//
// Precision: a top-K decision must not flip for score gaps above 1e-3, so a plain bf16
// product (error ~5e-4) is not enough.  Every fp32 operand is split into two bf16 terms,
// a = a_hi + a_lo with |a - a_hi - a_lo| <= 2^-18 |a|, and the contraction is
//     q.s_hi + q.s_lo + t_hi.s'_hi + t_hi.s'_lo + t_lo.s'_hi       (q is exact in bf16)
// on bf16 tensor cores with fp32 accumulation: ~1e-6 absolute score error.
//
// Kernels:
//   xw_mma_kernel    t = x W_down on tensor cores, stored as [t_hi | t_lo] bf16
//   sprep_kernel     per (h, c): [s_hi | s_lo | s'_hi | s'_lo] bf16 rows (the B operand)
// The contraction itself, with entropy, eligibility, the per-head scores and the group
// maximum zeta, is zeta_tc_kernel (score_tc.cuh, tcgen05 tensor cores).
#pragma once
#include "common.cuh"

namespace rdl {

// byte offset of 16-byte chunk `ch` in row `row` of a tile with `rowbytes`-byte rows,
// chunks XOR-swizzled within groups of 8 so 8 consecutive rows hit distinct banks
__device__ __forceinline__ uint32_t swz(int row, int ch, int rowbytes) {
  return (uint32_t)(row * rowbytes + ((ch ^ (row & 7)) << 4));
}

// --------------------------------------------------------------------------- t = x W_down
// CTA: 64 rows x all r columns (r <= 128, r % 16 == 0); 4 warps x 16 rows; K loop over D
// in blocks of 64 with double-buffered cp.async.  Output tt[row] = [t_hi (r) | t_lo (r)].
constexpr int XW_ROWS = 64, XW_KB = 64;

template <int R>
__global__ void __launch_bounds__(128) xw_mma_kernel(const __nv_bfloat16* __restrict__ x,
                                                     const __nv_bfloat16* __restrict__ w_down,
                                                     int M, int D,
                                                     __nv_bfloat16* __restrict__ tt) {
  constexpr int NT = R / 8;                       // n-tiles
  constexpr int WROW = R * 2;                     // bytes per W row (k) in smem
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char* Xs = smem_raw;                         // [2][64 rows][128 B]
  unsigned char* Ws = Xs + 2 * XW_ROWS * 128;           // [2][64 k][WROW]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int m0 = blockIdx.x * XW_ROWS;
  auto load = [&](int kb, int st) {
    const int k0 = kb * XW_KB;
    for (int e = tid; e < XW_ROWS * 8; e += 128) {
      const int r = e >> 3, ch = e & 7;
      const int gm = min(m0 + r, M - 1);
      cp_async16(smem_u32(Xs + st * XW_ROWS * 128 + swz(r, ch, 128)), x + (size_t)gm * D + k0 + ch * 8);
    }
    for (int e = tid; e < XW_KB * (R / 8); e += 128) {
      const int kr = e / (R / 8), ch = e % (R / 8);
      cp_async16(smem_u32(Ws + st * XW_KB * WROW + swz(kr, ch, WROW)), w_down + (size_t)(k0 + kr) * R + ch * 8);
    }
  };
  float acc[NT][4];
#pragma unroll
  for (int n = 0; n < NT; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
  const int nkb = D / XW_KB;
  load(0, 0);
  cp_async_commit();
  for (int kb = 0; kb < nkb; ++kb) {
    const int st = kb & 1;
    if (kb + 1 < nkb) load(kb + 1, st ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    const unsigned char* xs = Xs + st * XW_ROWS * 128;
    const unsigned char* ws = Ws + st * XW_KB * WROW;
#pragma unroll
    for (int ks = 0; ks < XW_KB / 16; ++ks) {
      uint32_t a[4];
      const int r = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1), ch = 2 * ks + (lane >> 4);
      ldsm_x4(smem_u32(xs + swz(r, ch, 128)), a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int n = 0; n < NT; n += 2) {
        // W stored [k][n]: transposed 8x8 loads give the k-major B fragment
        uint32_t b0, b1, b2, b3;
        const int jj = lane >> 3;
        const int kr = 16 * ks + 8 * (jj & 1) + (lane & 7), chn = n + (jj >> 1);
        ldsm_x4_t(smem_u32(ws + swz(kr, chn, WROW)), b0, b1, b2, b3);
        mma_bf16(acc[n], a, b0, b1);
        mma_bf16(acc[n + 1], a, b2, b3);
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  const int gq = lane >> 2, tq = lane & 3;
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int row = m0 + warp * 16 + gq + 8 * hr;
    if (row >= M) continue;
    __nv_bfloat16* o = tt + (size_t)row * (2 * R);
#pragma unroll
    for (int n = 0; n < NT; ++n) {
      const int col = n * 8 + 2 * tq;
      const float v0 = acc[n][2 * hr], v1 = acc[n][2 * hr + 1];
      const __nv_bfloat16 h0 = __float2bfloat16_rn(v0), h1 = __float2bfloat16_rn(v1);
      *reinterpret_cast<__nv_bfloat162*>(o + col) = __halves2bfloat162(h0, h1);
      *reinterpret_cast<__nv_bfloat162*>(o + R + col) = __halves2bfloat162(
          __float2bfloat16_rn(v0 - __bfloat162float(h0)), __float2bfloat16_rn(v1 - __bfloat162float(h1)));
    }
  }
}

// --------------------------------------------------------------------------- B operand rows
// SB[b,h,c] = [s_hi (128) | s_lo (128) | s'_hi (R) | s'_lo (R)] bf16, s' = W_up,h s.
// CTA per (32 chunks, head, batch); W_up,h staged in shared memory as fp32 (row pad +1).
template <int R>
__global__ void __launch_bounds__(256) sprep_kernel(const float* __restrict__ summary,
                                                    const __nv_bfloat16* __restrict__ w_up, int C,
                                                    int Hq, __nv_bfloat16* __restrict__ sb) {
  constexpr int D = 128, SBW = 2 * D + 2 * R;
  extern __shared__ float smf[];
  float* Wf = smf;                       // [R][D + 1]
  float* Sf = Wf + R * (D + 1);          // [8 warps][D]
  const int c0 = blockIdx.x * 32, h = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int e = tid; e < R * D; e += 256) {
    const int m = e / D, k = e % D;
    Wf[m * (D + 1) + k] = __bfloat162float(w_up[(size_t)m * Hq * D + (size_t)h * D + k]);
  }
  __syncthreads();
  float* sv = Sf + warp * D;
  for (int cc = warp; cc < 32; cc += 8) {
    const int c = c0 + cc;
    if (c >= C) break;
    const float* srow = summary + ((size_t)(b * Hq + h) * C + c) * D;
    __nv_bfloat16* o = sb + ((size_t)(b * Hq + h) * C + c) * SBW;
    for (int e = lane; e < D; e += 32) {
      const float s = srow[e];
      sv[e] = s;
      const __nv_bfloat16 hi = __float2bfloat16_rn(s);
      o[e] = hi;
      o[D + e] = __float2bfloat16_rn(s - __bfloat162float(hi));
    }
    __syncwarp();
    for (int m = lane; m < R; m += 32) {
      const float* wr = Wf + m * (D + 1);
      float acc = 0.f;
#pragma unroll 8
      for (int k = 0; k < D; ++k) acc = fmaf(wr[k], sv[k], acc);
      const __nv_bfloat16 hi = __float2bfloat16_rn(acc);
      o[2 * D + m] = hi;
      o[2 * D + R + m] = __float2bfloat16_rn(acc - __bfloat162float(hi));
    }
    __syncwarp();
  }
}

}  // namespace rdl
