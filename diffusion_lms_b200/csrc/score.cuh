// Route score, GQA group max and per-query top-K
// (Prefilling-dLLM v2, Figure 3 caption: "A content query adds a low-rank residual and
// scores these summaries.  Inside a GQA group the scores are reduced by a maximum, and
// the top K chunks are shared by every head in the group"; only remote chunks, i.e.
// chunks beyond the local window, are candidates -- Table 3).
//
// Three stages, all fp32 arithmetic so that selection decisions carry ~1e-6 score error:
//   1. t = x W_down, q_res = q + t W_up           (fp32 GEMMs, q_res kept in the workspace)
//   2. z[h,i,c] = tau q_res[i,h].s[h,c] - lambda H[h,c] (eligible c only), zeta = max over
//      the group's heads                           (tiled fp32 contraction, per group)
//   3. per (i, g): exact top-K of zeta (value desc, chunk asc), stored in ascending chunk
//      order, and the selected chunks' per-head scores gathered from z.
#pragma once
#include "common.cuh"

namespace rdl {

// --------------------------------------------------------------------------- stage 1
// Out[M,N] = A[M,Kd] * B[Kd,N] (+ Add[M,N]); fp32 accumulate and output.
template <typename TA, typename TB, typename TAdd>
__global__ void __launch_bounds__(256) gemm_f32_kernel(const TA* __restrict__ A,
                                                       const TB* __restrict__ Bm,
                                                       const TAdd* __restrict__ Add,
                                                       float* __restrict__ Out, int M, int N,
                                                       int Kd) {
  constexpr int BM = 64, BN = 64, BK = 16;
  __shared__ float As[BK][BM + 4];
  __shared__ float Bs[BK][BN + 4];
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const int m0 = blockIdx.y * BM, n0 = blockIdx.x * BN;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < Kd; k0 += BK) {
    for (int e = tid; e < BM * BK; e += 256) {
      const int r = e / BK, kk = e % BK;
      const int gm = m0 + r, gk = k0 + kk;
      As[kk][r] = (gm < M && gk < Kd) ? IO<TA>::ld(A + (size_t)gm * Kd + gk) : 0.f;
    }
    for (int e = tid; e < BK * BN; e += 256) {
      const int kk = e / BN, cc = e % BN;
      const int gk = k0 + kk, gn = n0 + cc;
      Bs[kk][cc] = (gk < Kd && gn < N) ? IO<TB>::ld(Bm + (size_t)gk * N + gn) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < BK; ++kk) {
      float a[4], bb[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) a[u] = As[kk][ty * 4 + u];
#pragma unroll
      for (int u = 0; u < 4; ++u) bb[u] = Bs[kk][tx * 4 + u];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int w = 0; w < 4; ++w) acc[u][w] = fmaf(a[u], bb[w], acc[u][w]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int gm = m0 + ty * 4 + u;
    if (gm >= M) continue;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int gn = n0 + tx * 4 + w;
      if (gn >= N) continue;
      float val = acc[u][w];
      if (Add) val += IO<TAdd>::ld(Add + (size_t)gm * N + gn);
      Out[(size_t)gm * N + gn] = val;
    }
  }
}

// Out[M,N] = A[M,Kd] * B[Kd,N] for few rows (decode blocks): one CTA per (row, 32 columns),
// the K loop split over 256 threads and reduced in shared memory.
template <typename TA, typename TB>
__global__ void __launch_bounds__(256) smallm_gemm_kernel(const TA* __restrict__ A,
                                                          const TB* __restrict__ Bm,
                                                          float* __restrict__ Out, int M, int N,
                                                          int Kd) {
  __shared__ float red[256][33];
  const int m = blockIdx.y, n0 = blockIdx.x * 32, tid = threadIdx.x;
  float acc[32];
#pragma unroll
  for (int j = 0; j < 32; ++j) acc[j] = 0.f;
  for (int k = tid; k < Kd; k += 256) {
    const float a = IO<TA>::ld(A + (size_t)m * Kd + k);
    const TB* br = Bm + (size_t)k * N + n0;
#pragma unroll
    for (int j = 0; j < 32; ++j) acc[j] = fmaf(a, (n0 + j < N) ? IO<TB>::ld(br + j) : 0.f, acc[j]);
  }
#pragma unroll
  for (int j = 0; j < 32; ++j) red[tid][j] = acc[j];
  __syncthreads();
  if (tid < 32) {
    float sum = 0.f;
    for (int t = 0; t < 256; ++t) sum += red[t][tid];
    if (n0 + tid < N) Out[(size_t)m * N + n0 + tid] = sum;
  }
}

// --------------------------------------------------------------------------- stage 2
// One CTA per (chunk tile of 64, query tile of 64, b*Hkv + g).
template <int D>
__global__ void __launch_bounds__(256) zeta_kernel(
    const float* __restrict__ qres, const int32_t* __restrict__ q_pos,
    const float* __restrict__ summary, const float* __restrict__ entropy, int Lq, int L, int Hq,
    int Hkv, int w, float lambda, float* __restrict__ z_all, float* __restrict__ zeta) {
  constexpr int BM = 64, BN = 64, BK = 16;
  __shared__ float Qs[BK][BM + 4];
  __shared__ float Ss[BK][BN + 4];
  __shared__ float Hs[BN];
  __shared__ int Ps[BM];
  const int C = L / S, G = Hq / Hkv;
  const int bg = blockIdx.z, b = bg / Hkv, g = bg % Hkv;
  const int i0 = blockIdx.y * BM, c0 = blockIdx.x * BN;
  const int tid = threadIdx.x, tx = tid % 16, ty = tid / 16;
  const float tau = rsqrtf((float)D);
  if (tid < BM) {
    const int i = i0 + tid;
    Ps[tid] = (i < Lq) ? (q_pos ? q_pos[(size_t)b * Lq + i] : i) : 0;
  }
  float zmax[4][4];
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v2 = 0; v2 < 4; ++v2) zmax[u][v2] = -INFINITY;

  for (int hl = 0; hl < G; ++hl) {
    const int h = g * G + hl;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < D; k0 += BK) {
      for (int e = tid; e < BM * BK; e += 256) {
        const int r = e / BK, kk = e % BK, i = i0 + r;
        Qs[kk][r] = (i < Lq) ? qres[((size_t)(b * Lq + i) * Hq + h) * D + k0 + kk] : 0.f;
      }
      for (int e = tid; e < BN * BK; e += 256) {
        const int cc = e / BK, kk = e % BK, c = c0 + cc;
        Ss[kk][cc] = (c < C) ? summary[((size_t)(b * Hq + h) * C + c) * D + k0 + kk] : 0.f;
      }
      if (k0 == 0 && tid < BN) {
        const int c = c0 + tid;
        Hs[tid] = (c < C) ? entropy[(size_t)(b * Hq + h) * C + c] : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < BK; ++kk) {
        float a[4], bb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) a[u] = Qs[kk][ty * 4 + u];
#pragma unroll
        for (int u = 0; u < 4; ++u) bb[u] = Ss[kk][tx * 4 + u];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int v2 = 0; v2 < 4; ++v2) acc[u][v2] = fmaf(a[u], bb[v2], acc[u][v2]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int r = ty * 4 + u, i = i0 + r;
      if (i >= Lq) continue;
      const int p = Ps[r];
#pragma unroll
      for (int v2 = 0; v2 < 4; ++v2) {
        const int cc = tx * 4 + v2, c = c0 + cc;
        if (c >= C) continue;
        const float z = chunk_eligible(c, p, w) ? tau * acc[u][v2] - lambda * Hs[cc] : -INFINITY;
        z_all[((size_t)(b * Hq + h) * Lq + i) * C + c] = z;
        zmax[u][v2] = fmaxf(zmax[u][v2], z);
      }
    }
    __syncthreads();   // Hs reloaded for the next head
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ty * 4 + u;
    if (i >= Lq) continue;
#pragma unroll
    for (int v2 = 0; v2 < 4; ++v2) {
      const int c = c0 + tx * 4 + v2;
      if (c < C) zeta[((size_t)(b * Hkv + g) * Lq + i) * C + c] = zmax[u][v2];
    }
  }
}

// --------------------------------------------------------------------------- stage 3
__device__ __forceinline__ bool better(float va, int ia, float vb, int ib) {
  return va > vb || (va == vb && ia < ib);
}

// One warp per (b, g, i).  Exact top-K (K <= 64) by K rounds of warp arg-max, ties to the
// smaller chunk index; selected chunks written in ascending order, then -1.
__global__ void __launch_bounds__(128) topk_kernel(const float* __restrict__ zeta,
                                                   const float* __restrict__ z_all,
                                                   const int32_t* __restrict__ q_pos, int Lq,
                                                   int L, int Hq, int Hkv, int K,
                                                   int32_t* __restrict__ idx,
                                                   float* __restrict__ z_sel) {
  extern __shared__ float zs[];
  const int C = L / S, G = Hq / Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long item = (long long)blockIdx.x * (blockDim.x / 32) + warp;
  if (item >= (long long)Lq * Hkv) return;
  const int b = blockIdx.y;
  const int g = (int)(item / Lq), i = (int)(item % Lq);
  float* row = zs + (size_t)warp * C;
  const int p = q_pos ? q_pos[(size_t)b * Lq + i] : i;
  int32_t* irow = idx + ((size_t)(b * Hkv + g) * Lq + i) * K;
  if (is_mask_slot(p)) {
    for (int k = lane; k < K; k += 32) {
      irow[k] = -1;
      for (int hl = 0; hl < G; ++hl) z_sel[((size_t)(b * Hq + g * G + hl) * Lq + i) * K + k] = -INFINITY;
    }
    return;
  }
  const float* zr = zeta + ((size_t)(b * Hkv + g) * Lq + i) * C;
  for (int c = lane; c < C; c += 32) row[c] = zr[c];
  __syncwarp();
  // each lane keeps the best of its strided elements
  auto scan = [&](float& bv, int& bi) {
    bv = -INFINITY;
    bi = 0x7fffffff;
    for (int c = lane; c < C; c += 32) {
      const float vv = row[c];
      if (vv > bv) { bv = vv; bi = c; }
    }
  };
  float bv;
  int bi;
  scan(bv, bi);
  int sel0 = -1, sel1 = -1;   // lane k holds selection k (and k + 32)
  for (int k = 0; k < K; ++k) {
    float wv = bv;
    int wi = bi;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, wv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, wi, o);
      if (better(ov, oi, wv, wi)) { wv = ov; wi = oi; }
    }
    if (wv == -INFINITY) break;           // no eligible chunk left
    if (lane == (k & 31)) { if (k < 32) sel0 = wi; else sel1 = wi; }
    if (lane == (wi & 31)) {              // owner of the winner removes it and rescans
      row[wi] = -INFINITY;
      scan(bv, bi);
    }
    __syncwarp();
  }
  // ascending order: rank of each selected index among the valid selections
  const int BIG = 0x7fffffff;
  const int key0 = sel0 < 0 ? BIG : sel0, key1 = sel1 < 0 ? BIG : sel1;
  int rank0 = 0, rank1 = 0;
  for (int k = 0; k < K; ++k) {
    const int src = __shfl_sync(0xffffffffu, k < 32 ? key0 : key1, k & 31);
    rank0 += (src < key0);
    rank1 += (src < key1);
  }
  const int slot0 = lane, slot1 = lane + 32;
  if (slot0 < K && sel0 >= 0) irow[rank0] = sel0;
  if (slot1 < K && sel1 >= 0) irow[rank1] = sel1;
  // count valid selections to fill the -1 tail
  int nvalid = 0;
  for (int k = 0; k < K; ++k) {
    const int src = __shfl_sync(0xffffffffu, k < 32 ? key0 : key1, k & 31);
    nvalid += (src != BIG);
  }
  for (int k = nvalid + lane; k < K; k += 32) irow[k] = -1;
  __syncwarp();
  // per-head scores of the selected chunks
  for (int e = lane; e < K * G; e += 32) {
    const int k = e % K, hl = e / K, h = g * G + hl;
    const int c = (k < nvalid) ? irow[k] : -1;
    const float zz = (c >= 0) ? z_all[((size_t)(b * Hq + h) * Lq + i) * C + c] : -INFINITY;
    z_sel[((size_t)(b * Hq + h) * Lq + i) * K + k] = zz;
  }
}

}  // namespace rdl
