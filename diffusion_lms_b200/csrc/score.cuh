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

namespace rdl {

// --------------------------------------------------------------------------- radix top-K
// Order-preserving map float -> uint32 (larger float, larger key; -inf lowest finite-less).
__device__ __forceinline__ uint32_t order_key(float f) {
  const uint32_t b = __float_as_uint(f);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

// One warp per (b, g, i): exact top-K of zeta over the row, ties to the smaller chunk index,
// the selection in ascending chunk order; then the per-head scores of the selected chunks are
// gathered.  Candidate filter first: with packed keys (order key << 32 | ~chunk, distinct per
// chunk), every lane holds ceil(K/32) keys at or above its ceil(K/32)-th largest, so the
// smallest of those over the warp bounds the K-th largest key from below and only the keys at
// or above it (typically a few K) are ranked exactly.  When more than TK_MAXCAND keys pass
// (heavy near-ties), or the row is short (C < TK_FILTER_MINC), a 4-pass 8-bit radix select finds the K-th largest key and one in-order
// pass takes every key above it and the first (by chunk index) of the keys equal to it.
constexpr int TK_MAXCAND = 256;
constexpr int TK_FILTER_MINC = 512;   // below this many chunks the radix select is faster (measured)
// shared memory words per warp of topk_radix_kernel: keys [C], then (8-byte aligned) the
// radix histogram or the packed candidates
__host__ __device__ inline int topk_warp_words(int C) { return ((C + 1) & ~1) + 2 * TK_MAXCAND; }

__global__ void __launch_bounds__(128) topk_radix_kernel(const float* __restrict__ zeta,
                                                         const float* __restrict__ z_all,
                                                         const int32_t* __restrict__ q_pos, int Lq,
                                                         int L, int Hq, int Hkv, int K,
                                                         int32_t* __restrict__ idx,
                                                         float* __restrict__ z_sel) {
  extern __shared__ uint32_t tk_smem[];
  const int C = L / S, G = Hq / Hkv;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const long long item = (long long)blockIdx.x * (blockDim.x / 32) + warp;
  if (item >= (long long)Lq * Hkv) return;
  const int b = blockIdx.y;
  const int g = (int)(item / Lq), i = (int)(item % Lq);
  uint32_t* keys = tk_smem + (size_t)warp * topk_warp_words(C);
  uint32_t* hist = keys + ((C + 1) & ~1);
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
  const uint32_t kneg = order_key(-INFINITY);
  auto packed = [](uint32_t k, int cc) -> unsigned long long {
    return ((unsigned long long)k << 32) | (0xffffffffu - (uint32_t)cc);
  };
  int nvalid = 0;
  unsigned long long m1 = 0ull, m2 = 0ull;     // the lane's two largest packed keys
  auto track = [&](uint32_t k, int cc) {
    if (k > kneg) {
      ++nvalid;
      const unsigned long long pk = packed(k, cc);
      if (pk > m1) { m2 = m1; m1 = pk; } else if (pk > m2) { m2 = pk; }
    }
  };
  int c = lane;
  for (; c + 7 * 32 < C; c += 8 * 32) {      // 8 independent loads in flight per lane
    float zv[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) zv[u] = zr[c + 32 * u];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const uint32_t k = order_key(zv[u]);
      keys[c + 32 * u] = k;
      track(k, c + 32 * u);
    }
  }
  for (; c < C; c += 32) {
    const uint32_t k = order_key(zr[c]);
    keys[c] = k;
    track(k, c);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) nvalid += __shfl_xor_sync(0xffffffffu, nvalid, o);
  __syncwarp();
  int nsel = -1;           // set by the candidate filter when it decides the row
  if (nvalid > K && K <= 64 && C >= TK_FILTER_MINC) {
    unsigned long long t0 = K <= 32 ? m1 : m2;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const unsigned long long y = __shfl_xor_sync(0xffffffffu, t0, o);
      t0 = y < t0 ? y : t0;
    }
    // t0 = 0 when a lane holds too few valid keys: then every valid key is a candidate
    int cnt = 0;
    for (int cc = lane; cc < C; cc += 32) {
      const uint32_t k = keys[cc];
      cnt += (k > kneg && packed(k, cc) >= t0);
    }
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const int total = __shfl_sync(0xffffffffu, incl, 31);
    if (total <= TK_MAXCAND) {
      unsigned long long* cand = reinterpret_cast<unsigned long long*>(hist);
      int pos = incl - cnt;
      for (int cc = lane; cc < C; cc += 32) {
        const uint32_t k = keys[cc];
        if (k > kneg) {
          const unsigned long long pk = packed(k, cc);
          if (pk >= t0) cand[pos++] = pk;
        }
      }
      __syncwarp();
      // exact rank of each candidate (packed keys are distinct); the K best by rank into
      // selr[0 .. K), then into ascending chunk order
      int* selr = reinterpret_cast<int*>(keys);     // the keys are no longer read
      for (int j = lane; j < total; j += 32) {
        const unsigned long long mine = cand[j];
        int rank = 0;
        for (int m = 0; m < total; ++m) rank += cand[m] > mine;
        if (rank < K) selr[rank] = (int)(0xffffffffu - (uint32_t)(mine & 0xffffffffull));
      }
      __syncwarp();
      for (int j = lane; j < K; j += 32) {
        const int cj = selr[j];
        int at = 0;
        for (int m = 0; m < K; ++m) at += selr[m] < cj;
        irow[at] = cj;
      }
      __syncwarp();
      nsel = K;
    }
  }
  uint32_t thr = kneg;     // take keys > thr, plus `need` keys == thr (smallest indices)
  int need = 0;
  if (nsel < 0 && nvalid > K) {
    uint32_t prefix = 0, pmask = 0;
    need = K;
    for (int shift = 24; shift >= 0; shift -= 8) {
#pragma unroll
      for (int u = 0; u < 8; ++u) hist[lane * 8 + u] = 0;
      __syncwarp();
      // scores cluster in a few digits (same sign/exponent): aggregate lanes that hit the
      // same bin so each bin takes one atomic per step
      for (int base = 0; base < C; base += 32) {
        const int c = base + lane;
        const uint32_t k = c < C ? keys[c] : 0u;
        const bool in = c < C && (k & pmask) == prefix;
        const unsigned dig = in ? ((k >> shift) & 255u) : 256u;
        const unsigned peers = __match_any_sync(0xffffffffu, dig);
        if (in && lane == __ffs(peers) - 1) atomicAdd(&hist[dig], (unsigned)__popc(peers));
      }
      __syncwarp();
      // lane owns bins [8*lane, 8*lane+8); count of matching keys in bins above each lane
      int local = 0;
#pragma unroll
      for (int u = 0; u < 8; ++u) local += (int)hist[lane * 8 + u];
      // walk the lanes from the top bin down to the lane holding the need-th key
      int incl = 0, target_lane = -1, excl_at_target = 0;
      for (int l2 = 31; l2 >= 0; --l2) {
        const int v = __shfl_sync(0xffffffffu, local, l2);
        if (target_lane < 0 && incl + v >= need) { target_lane = l2; excl_at_target = incl; }
        incl += v;
      }
      int digit = 0, cnt_above = excl_at_target;
      if (lane == target_lane) {
        int run = excl_at_target;
        for (int u = 7; u >= 0; --u) {
          const int v = (int)hist[lane * 8 + u];
          if (run + v >= need) { digit = lane * 8 + u; cnt_above = run; break; }
          run += v;
        }
      }
      digit = __shfl_sync(0xffffffffu, digit, target_lane);
      cnt_above = __shfl_sync(0xffffffffu, cnt_above, target_lane);
      need -= cnt_above;
      prefix |= (uint32_t)digit << shift;
      pmask |= 255u << shift;
      __syncwarp();
    }
    thr = prefix;
  }
  // in-order selection (unless the candidate filter decided the row)
  if (nsel < 0) {
  int taken = 0, ties = 0;
  const unsigned lt = (1u << lane) - 1u;
  for (int base = 0; base < C; base += 32) {
    const int c = base + lane;
    const uint32_t k = c < C ? keys[c] : 0u;
    const bool tie = c < C && need > 0 && k == thr;
    const unsigned tmask = __ballot_sync(0xffffffffu, tie);
    const bool take = (c < C && k > thr) || (tie && ties + __popc(tmask & lt) < need);
    ties += __popc(tmask);
    const unsigned smask = __ballot_sync(0xffffffffu, take);
    if (take) {
      const int pos = taken + __popc(smask & lt);
      if (pos < K) irow[pos] = c;
    }
    taken += __popc(smask);
  }
  for (int k = taken + lane; k < K; k += 32) irow[k] = -1;
  __syncwarp();
  nsel = taken < K ? taken : K;
  }
  // per-head scores of the selection (without z_all they come later, from the scorer's second
  // pass over the selected chunks; every slot starts at -inf)
  for (int e = lane; e < K * G; e += 32) {
    const int k = e % K, hl = e / K, h = g * G + hl;
    const int c = (k < nsel) ? irow[k] : -1;
    z_sel[((size_t)(b * Hq + h) * Lq + i) * K + k] =
        (c >= 0 && z_all) ? z_all[((size_t)(b * Hq + h) * Lq + i) * C + c] : -INFINITY;
  }
}

}  // namespace rdl

namespace rdl {

// Block-wide exclusive scan of one int per thread (256 threads); returns the total.
__device__ __forceinline__ int block_excl_scan256(int v, int* warp_sums, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  int base = 0, tot = 0;
#pragma unroll
  for (int w8 = 0; w8 < 8; ++w8) {
    const int ws = warp_sums[w8];
    if (w8 < warp) base += ws;
    tot += ws;
  }
  __syncthreads();
  total = tot;
  return base + x - v;
}

// Block-wide exclusive scan of one int per thread (NT threads); returns the total.
template <int NT>
__device__ __forceinline__ int block_excl_scan_t(int v, int* warp_sums, int& total) {
  constexpr int NW = NT / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  int base = 0, tot = 0;
#pragma unroll
  for (int w8 = 0; w8 < NW; ++w8) {
    const int ws = warp_sums[w8];
    if (w8 < warp) base += ws;
    tot += ws;
  }
  __syncthreads();
  total = tot;
  return base + x - v;
}

// Exact top-K of the order keys keys[0..C) by one CTA of NT threads (NT >= 256): a 4-pass
// 8-bit radix select for the K-th largest key, then an in-order compaction that takes every
// key above it and the first (by chunk index) of the keys equal to it.  sel_s receives the
// selected chunk indices in ascending order; returns how many there are (min(#valid, K)).
// whist: NT/32 per-warp histograms of 256 bins; warp_sums: NT/32 ints.
template <int NT>
__device__ __forceinline__ int cta_select_topk_t(const uint32_t* keys, int C, int K, unsigned* hist,
                                                 unsigned (*whist)[256], int* warp_sums, int* bc, int* sel_s) {
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t kneg = order_key(-INFINITY);
  int nv = 0;
  for (int c = tid; c < C; c += NT) nv += keys[c] > kneg;
  int nvalid;
  (void)block_excl_scan_t<NT>(nv, warp_sums, nvalid);
  uint32_t thr = kneg;
  int need = 0;
  if (nvalid > K) {
    uint32_t prefix = 0, pmask = 0;
    need = K;
    for (int shift = 24; shift >= 0; shift -= 8) {
      // per-warp histograms: no two warps contend for one bin (the keys cluster in a few
      // digits, so a shared histogram would serialise the whole CTA on those bins)
#pragma unroll
      for (int u = 0; u < 8; ++u) whist[warp][lane * 8 + u] = 0;
      __syncwarp();
      for (int base = 0; base < C; base += NT) {
        const int c = base + tid;
        const uint32_t k = c < C ? keys[c] : 0u;
        if (c < C && (k & pmask) == prefix) atomicAdd(&whist[warp][(k >> shift) & 255u], 1u);
      }
      __syncwarp();
      __syncthreads();
      if (tid < 256) {
        unsigned sum = 0;
#pragma unroll
        for (int w8 = 0; w8 < NW; ++w8) sum += whist[w8][tid];
        hist[tid] = sum;
      }
      __syncthreads();
      if (warp == 0) {
        // lane l owns bins 255-8l .. 248-8l (largest digits first); an inclusive warp scan
        // of the lane counts finds the lane holding the need-th largest key
        int cnt[8], local = 0;
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          cnt[u] = (int)hist[255 - 8 * lane - u];
          local += cnt[u];
        }
        int incl = local;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += y;
        }
        const unsigned hit = __ballot_sync(0xffffffffu, incl >= need);
        if (lane == __ffs(hit) - 1) {
          int run = incl - local, dg = 0, ca = run;
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            if (run + cnt[u] >= need) { dg = 255 - 8 * lane - u; ca = run; break; }
            run += cnt[u];
          }
          bc[0] = dg;
          bc[1] = ca;
        }
      }
      __syncthreads();
      need -= bc[1];
      prefix |= (uint32_t)bc[0] << shift;
      pmask |= 255u << shift;
      __syncthreads();
    }
    thr = prefix;
  }
  // ordered compaction: thread t owns the contiguous range [t*seg, (t+1)*seg)
  const int seg = (C + NT - 1) / NT, c0 = tid * seg, c1 = min(C, c0 + seg);
  int ngt = 0, nties = 0;
  for (int c = c0; c < c1; ++c) {
    const uint32_t k = keys[c];
    ngt += k > thr;
    nties += (need > 0 && k == thr);
  }
  int tot;
  const int tie_base = block_excl_scan_t<NT>(nties, warp_sums, tot);
  const int take_ties = max(0, min(nties, need - tie_base));
  const int pos0 = block_excl_scan_t<NT>(ngt + take_ties, warp_sums, tot);
  int pos = pos0, tk = 0;
  for (int c = c0; c < c1; ++c) {
    const uint32_t k = keys[c];
    bool take = k > thr;
    if (!take && need > 0 && k == thr && tk < take_ties) { take = true; ++tk; }
    if (take && pos < K) sel_s[pos] = c;
    pos += take;
  }
  __syncthreads();
  return min(tot, K);
}
__device__ __forceinline__ int cta_select_topk(const uint32_t* keys, int C, int K, unsigned* hist,
                                               unsigned (*whist)[256], int* warp_sums, int* bc, int* sel_s) {
  return cta_select_topk_t<256>(keys, C, K, hist, whist, warp_sums, bc, sel_s);
}

// One CTA (256 threads) per (b, g, i): the same exact top-K as topk_radix_kernel, for few
// rows over many chunks (decode blocks).  Keys are split across the CTA; the selection is
// compacted in chunk order with block scans.
__global__ void __launch_bounds__(256) topk_cta_kernel(const float* __restrict__ zeta,
                                                       const float* __restrict__ z_all,
                                                       const int32_t* __restrict__ q_pos, int Lq, int L,
                                                       int Hq, int Hkv, int K, int32_t* __restrict__ idx,
                                                       float* __restrict__ z_sel) {
  extern __shared__ uint32_t tc_keys[];
  __shared__ unsigned hist[256];
  __shared__ unsigned whist[8][256];
  __shared__ int warp_sums[8];
  __shared__ int sel_s[64];
  __shared__ int bc[3];
  const int C = L / S, G = Hq / Hkv;
  const int tid = threadIdx.x;
  const int item = blockIdx.x, b = blockIdx.y;
  const int g = item / Lq, i = item % Lq;
  const int p = q_pos ? q_pos[(size_t)b * Lq + i] : i;
  int32_t* irow = idx + ((size_t)(b * Hkv + g) * Lq + i) * K;
  if (is_mask_slot(p)) {
    for (int e = tid; e < K * G; e += 256) {
      const int k = e % K, hl = e / K;
      if (hl == 0) irow[k] = -1;
      z_sel[((size_t)(b * Hq + g * G + hl) * Lq + i) * K + k] = -INFINITY;
    }
    return;
  }
  const float* zr = zeta + ((size_t)(b * Hkv + g) * Lq + i) * C;
  for (int c = tid; c < C; c += 256) tc_keys[c] = order_key(zr[c]);
  __syncthreads();
  const int nsel = cta_select_topk(tc_keys, C, K, hist, whist, warp_sums, bc, sel_s);
  for (int e = tid; e < K * G; e += 256) {
    const int k = e % K, hl = e / K, h = g * G + hl;
    const int c = k < nsel ? sel_s[k] : -1;
    if (hl == 0) irow[k] = c;
    z_sel[((size_t)(b * Hq + h) * Lq + i) * K + k] =
        (c >= 0 && z_all) ? z_all[((size_t)(b * Hq + h) * Lq + i) * C + c] : -INFINITY;
  }
}

}  // namespace rdl
