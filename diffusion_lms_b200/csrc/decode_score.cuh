// Route score for decode blocks (few query rows over a long cached context).
//
// Same definition as the prefill scorer ([v2] Figure 3: residual-adapted content queries
// score the summaries, the pooling entropy enters with weight lambda, the group max picks
// the chunks), organised for the decode shape: the summaries s [Hq, C, d] (fp32, cached
// across decode steps) dominate the bytes, so they are streamed from HBM exactly once.
//
//   dec_tpart/dec_tsum/dec_qres   q_res = q + (x W_down) W_up for each row (fp32): the
//                        weights are read once, slice by slice
//   decode_score_kernel  per (64-chunk tile, KV group): for each head, the fp32 summaries
//                        and residual queries are split into bf16 hi/lo terms in shared
//                        memory and contracted on tensor cores,
//                        q_hi.s_hi + q_hi.s_lo + q_lo.s_hi  (~1e-6 absolute error),
//                        then entropy, eligibility, per-head scores and the group max.
#pragma once
#include "common.cuh"

namespace rdl {

// --------------------------------------------------------------------------- q_res, sliced
// For few rows the weights dominate the bytes, so each CTA reads one slice of them once:
//   dec_tpart_kernel  partial t over a 128-wide slice of D for up to 64 rows (grid: slices)
//   dec_tsum_kernel   t = sum of the slice partials
//   dec_qres_kernel   q_res = q + t W_up for one 128-wide column block (grid: column blocks)
constexpr int DQ_ROWS = 64, DQ_KS = 64;
constexpr int DQ_TPART_SMEM = (DQ_ROWS * (DQ_KS + 1) + DQ_KS * (128 + 1)) * 4;
constexpr int DQ_QRES_SMEM = (DQ_ROWS * (128 + 1) + 128 * (128 + 1)) * 4;

template <typename T>
__global__ void __launch_bounds__(256) dec_tpart_kernel(const T* __restrict__ x, const T* __restrict__ w_down,
                                                        int M, int D, int r, float* __restrict__ tpart) {
  extern __shared__ float dq_smem[];
  float (*xs)[DQ_KS + 1] = reinterpret_cast<float (*)[DQ_KS + 1]>(dq_smem);
  float (*ws)[128 + 1] = reinterpret_cast<float (*)[128 + 1]>(dq_smem + DQ_ROWS * (DQ_KS + 1));
  const int slice = blockIdx.x, m0 = blockIdx.y * DQ_ROWS, tid = threadIdx.x;
  const int k0 = slice * DQ_KS, kn = min(DQ_KS, D - k0);
  for (int e = tid; e < DQ_ROWS * DQ_KS; e += 256) {
    const int rr = e / DQ_KS, kk = e % DQ_KS;
    xs[rr][kk] = (m0 + rr < M && kk < kn) ? IO<T>::ld(x + (size_t)(m0 + rr) * D + k0 + kk) : 0.f;
  }
  for (int e = tid; e < DQ_KS * r; e += 256) {
    const int kk = e / r, m = e % r;
    ws[kk][m] = kk < kn ? IO<T>::ld(w_down + (size_t)(k0 + kk) * r + m) : 0.f;
  }
  __syncthreads();
  // thread: 4 rows x (r/16) columns
  const int tr = tid / 16, tc = tid % 16;      // rows tr*4.., columns tc + 16*j
  const int nc = (r + 15) / 16;
  float acc[4][8];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[a][j] = 0.f;
  for (int kk = 0; kk < DQ_KS; ++kk) {
    float xv[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) xv[a] = xs[tr * 4 + a][kk];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      if (j >= nc) break;
      const float wv = ws[kk][tc + 16 * j];
#pragma unroll
      for (int a = 0; a < 4; ++a) acc[a][j] = fmaf(xv[a], wv, acc[a][j]);
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int row = m0 + tr * 4 + a;
    if (row >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int m = tc + 16 * j;
      if (j < nc && m < r) tpart[((size_t)slice * M + row) * r + m] = acc[a][j];
    }
  }
}

__global__ void dec_tsum_kernel(const float* __restrict__ tpart, int nslices, int n, float* __restrict__ t) {
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n) return;
  float s[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  int sl = 0;
  for (; sl + 8 <= nslices; sl += 8) {
#pragma unroll
    for (int u = 0; u < 8; ++u) s[u] += tpart[(size_t)(sl + u) * n + e];
  }
  for (; sl < nslices; ++sl) s[0] += tpart[(size_t)sl * n + e];
  t[e] = ((s[0] + s[1]) + (s[2] + s[3])) + ((s[4] + s[5]) + (s[6] + s[7]));
}

template <typename T>
__global__ void __launch_bounds__(256) dec_qres_kernel(const T* __restrict__ q, const float* __restrict__ t,
                                                       const T* __restrict__ w_up, int M, int r, int HD,
                                                       float* __restrict__ qres) {
  extern __shared__ float dq_smem[];
  float (*ts)[128 + 1] = reinterpret_cast<float (*)[128 + 1]>(dq_smem);
  float (*ws)[128 + 1] = reinterpret_cast<float (*)[128 + 1]>(dq_smem + DQ_ROWS * (128 + 1));
  const int c0 = blockIdx.x * 128, m0 = blockIdx.y * DQ_ROWS, tid = threadIdx.x;
  const int cn = min(128, HD - c0);
  for (int e = tid; e < DQ_ROWS * r; e += 256) {
    const int rr = e / r, m = e % r;
    ts[rr][m] = (m0 + rr < M && t) ? t[(size_t)(m0 + rr) * r + m] : 0.f;
  }
  for (int e = tid; e < r * 128; e += 256) {
    const int m = e / 128, cc = e % 128;
    ws[m][cc] = cc < cn ? IO<T>::ld(w_up + (size_t)m * HD + c0 + cc) : 0.f;
  }
  __syncthreads();
  const int tr = tid / 16, tc = tid % 16;      // rows tr*4.., columns tc + 16*j (8 columns)
  float acc[4][8];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int row = m0 + tr * 4 + a, col = c0 + tc + 16 * j;
      acc[a][j] = (row < M && col < HD) ? IO<T>::ld(q + (size_t)row * HD + col) : 0.f;
    }
  for (int m = 0; m < r; ++m) {
    float tv[4];
#pragma unroll
    for (int a = 0; a < 4; ++a) tv[a] = ts[tr * 4 + a][m];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const float wv = ws[m][tc + 16 * j];
#pragma unroll
      for (int a = 0; a < 4; ++a) acc[a][j] = fmaf(tv[a], wv, acc[a][j]);
    }
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int row = m0 + tr * 4 + a;
    if (row >= M) continue;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int col = c0 + tc + 16 * j;
      if (col < HD) qres[(size_t)row * HD + col] = acc[a][j];
    }
  }
}

// --------------------------------------------------------------------------- scores
constexpr int DS_CH = 64;     // chunks per CTA
constexpr int DS_ROWS = 32;   // query rows per pass (decode blocks have at most 63 rows)
constexpr int DS_SMEM = DS_ROWS * 512 + DS_CH * 512;

// byte offset of 16-byte chunk `ch` of row `row` in a tile of 512-byte rows
// ([hi 128 | lo 128] bf16), chunks XOR-swizzled within groups of 8
__device__ __forceinline__ uint32_t swz512(int row, int ch) {
  return (uint32_t)(row * 512 + ((ch ^ (row & 7)) << 4));
}

// fp32 row of 128 -> [hi (128) | lo (128)] bf16 in a swizzled 512-byte smem row
__device__ __forceinline__ void split_row_store(unsigned char* tile, int row, int ch8, const float* f) {
  uint32_t hi[4], lo[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const __nv_bfloat16 h0 = __float2bfloat16_rn(f[2 * u]), h1 = __float2bfloat16_rn(f[2 * u + 1]);
    const __nv_bfloat162 hh = __halves2bfloat162(h0, h1);
    const __nv_bfloat162 ll = __floats2bfloat162_rn(f[2 * u] - __bfloat162float(h0),
                                                    f[2 * u + 1] - __bfloat162float(h1));
    hi[u] = *reinterpret_cast<const uint32_t*>(&hh);
    lo[u] = *reinterpret_cast<const uint32_t*>(&ll);
  }
  *reinterpret_cast<uint4*>(tile + swz512(row, ch8)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
  *reinterpret_cast<uint4*>(tile + swz512(row, 16 + ch8)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
}

// grid (ceil(C/64), B*Hkv); 128 threads = 4 warps in a 2 x 2 grid of 16 rows x 32 chunks.
__global__ void __launch_bounds__(128) decode_score_kernel(
    const float* __restrict__ qres, const int32_t* __restrict__ q_pos, const float* __restrict__ summary,
    const float* __restrict__ entropy, int Lq, int L, int Hq, int Hkv, int w, float lambda,
    float* __restrict__ z_all, float* __restrict__ zeta) {
  constexpr int D = 128;
  extern __shared__ __align__(128) unsigned char ds_smem[];
  unsigned char* Qs = ds_smem;                  // [32 rows][512 B]  16 KB
  unsigned char* Ss = ds_smem + DS_ROWS * 512;  // [64 chunks][512 B] 32 KB
  __shared__ float Hs[DS_CH];
  __shared__ int Ps[DS_ROWS];
  const int C = L / S, G = Hq / Hkv;
  const int bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv;
  const int c0 = blockIdx.x * DS_CH;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int wm = warp >> 1, wn = warp & 1;
  const int gq = lane >> 2, tq = lane & 3;
  const float tau = rsqrtf((float)D);

  for (int r0 = 0; r0 < Lq; r0 += DS_ROWS) {
    __syncthreads();   // the previous pass has finished reading Ps
    if (tid < DS_ROWS) {
      const int i = r0 + tid;
      Ps[tid] = (i < Lq) ? (q_pos ? q_pos[(size_t)b * Lq + i] : i) : INT_MIN;
    }
    float zmax[4][4];
#pragma unroll
    for (int n = 0; n < 4; ++n) zmax[n][0] = zmax[n][1] = zmax[n][2] = zmax[n][3] = -INFINITY;
    for (int hl = 0; hl < G; ++hl) {
      const int h = g * G + hl;
      __syncthreads();   // previous head's tiles fully consumed
      // stage q_res rows and summaries of this head as bf16 hi/lo; all loads of a thread
      // are issued before any conversion so they are in flight together
      {
        constexpr int NQ = DS_ROWS * 16 / 128, NS = DS_CH * 16 / 128;
        float fq[NQ][8], fs[NS][8];
#pragma unroll
        for (int u = 0; u < NQ; ++u) {
          const int e = tid + 128 * u, rr = e >> 4, ch8 = e & 15, i = min(r0 + rr, Lq - 1);
          load8(qres + ((size_t)(b * Lq + i) * Hq + h) * D + ch8 * 8, fq[u]);
        }
#pragma unroll
        for (int u = 0; u < NS; ++u) {
          const int e = tid + 128 * u, cc = e >> 4, ch8 = e & 15, c = min(c0 + cc, C - 1);
          load8(summary + ((size_t)(b * Hq + h) * C + c) * D + ch8 * 8, fs[u]);
        }
#pragma unroll
        for (int u = 0; u < NQ; ++u) {
          const int e = tid + 128 * u;
          split_row_store(Qs, e >> 4, e & 15, fq[u]);
        }
#pragma unroll
        for (int u = 0; u < NS; ++u) {
          const int e = tid + 128 * u;
          split_row_store(Ss, e >> 4, e & 15, fs[u]);
        }
      }
      if (tid < DS_CH) Hs[tid] = (c0 + tid < C) ? entropy[(size_t)(b * Hq + h) * C + c0 + tid] : 0.f;
      __syncthreads();
      float acc[4][4];
#pragma unroll
      for (int n = 0; n < 4; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
      // (q_hi, s_hi), (q_hi, s_lo), (q_lo, s_hi): A chunk base 0/0/16, B chunk base 0/16/0
#pragma unroll
      for (int part = 0; part < 3; ++part) {
        const int abase = part == 2 ? 16 : 0, bbase = part == 1 ? 16 : 0;
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          uint32_t a[4];
          const int ra = wm * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
          ldsm_x4(smem_u32(Qs + swz512(ra, abase + 2 * ks + (lane >> 4))), a[0], a[1], a[2], a[3]);
#pragma unroll
          for (int np = 0; np < 4; np += 2) {
            uint32_t b0, b1, b2, b3;
            const int rb = wn * 32 + np * 8 + (lane & 7) + 8 * (lane >> 4);
            ldsm_x4(smem_u32(Ss + swz512(rb, bbase + 2 * ks + ((lane >> 3) & 1))), b0, b1, b2, b3);
            mma_bf16(acc[np], a, b0, b1);
            mma_bf16(acc[np + 1], a, b2, b3);
          }
        }
      }
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int rl = wm * 16 + gq + 8 * hr, i = r0 + rl;
        const int p = Ps[rl];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
#pragma unroll
          for (int e2 = 0; e2 < 2; ++e2) {
            const int cc = wn * 32 + n * 8 + 2 * tq + e2, c = c0 + cc;
            const float z = (c < C && chunk_eligible(c, p, w)) ? tau * acc[n][2 * hr + e2] - lambda * Hs[cc]
                                                               : -INFINITY;
            zmax[n][2 * hr + e2] = fmaxf(zmax[n][2 * hr + e2], z);
            if (i < Lq && c < C) z_all[((size_t)(b * Hq + h) * Lq + i) * C + c] = z;
          }
        }
      }
    }
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int i = r0 + wm * 16 + gq + 8 * hr;
      if (i >= Lq) continue;
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
          const int c = c0 + wn * 32 + n * 8 + 2 * tq + e2;
          if (c < C) zeta[((size_t)(b * Hkv + g) * Lq + i) * C + c] = zmax[n][2 * hr + e2];
        }
    }
  }
}

}  // namespace rdl
