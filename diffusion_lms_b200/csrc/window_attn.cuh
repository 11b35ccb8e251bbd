// Bidirectional local-window attention: the non-route layers' sliding window and the
// route layer's local window (Prefilling-dLLM v2 abstract: "a query keeps a bidirectional
// local window ... the other layers use a bidirectional sliding window"; radius per
// Table 3).  W(p) = { j : |p - j| <= w, 0 <= j < L }, every slot included.
//
// generic_attn_kernel: scalar fp32 kernel for any dtype / head dim, computing either the
//   sliding-window output or the whole two-level route partition in one pass.
// window_mma_kernel:   bf16, d = 128 banded flash kernel on mma.sync tensor cores, used
//   when the keys of a row tile are split over several CTAs (few query rows) or a group
//   has more than 8 heads; otherwise window_tc.cuh runs the window on tcgen05.
//   CTA = 16 consecutive query rows x one KV group; warp w = head w of the group, so the
//   window's K/V tiles (64 keys, double-buffered via cp.async) are shared by every head.
#pragma once
#include "common.cuh"

namespace rdl {

// --------------------------------------------------------------------------- generic
// Online (m, l, acc) over a key range of one KV head; lanes split keys for the logits
// and the head dim for the accumulation.
template <typename T, int D>
__device__ void attend_range(const float* qs, const T* __restrict__ kg, const T* __restrict__ vg,
                             int j0, int j1, float& m, float& l, float* acc, int lane) {
  constexpr int EPL = D / 32;
  const float tau = rsqrtf((float)D);
  for (int jb = j0; jb < j1; jb += 32) {
    const int j = jb + lane;
    float logit = -INFINITY;
    if (j < j1) {
      const T* kr = kg + (size_t)j * D;
      float dot = 0.f;
#pragma unroll 8
      for (int e = 0; e < D; ++e) dot = fmaf(qs[e], IO<T>::ld(kr + e), dot);
      logit = dot * tau;
    }
    const float bm = warp_max(logit);
    const float mn = fmaxf(m, bm);
    const float alpha = (m == -INFINITY) ? 0.f : expf(m - mn);
    const float pj = (j < j1) ? expf(logit - mn) : 0.f;
    l = l * alpha + warp_sum(pj);
#pragma unroll
    for (int u = 0; u < EPL; ++u) acc[u] *= alpha;
    const int nj = min(32, j1 - jb);
    for (int t = 0; t < nj; ++t) {
      const float pt = __shfl_sync(0xffffffffu, pj, t);
      const T* vr = vg + (size_t)(jb + t) * D;
#pragma unroll
      for (int u = 0; u < EPL; ++u) acc[u] = fmaf(pt, IO<T>::ld(vr + lane + 32 * u), acc[u]);
    }
    m = mn;
  }
}

// grid (Lq, Hkv, B), 128 threads; warp loops over the group's heads.
template <typename T, int D, bool ROUTE>
__global__ void __launch_bounds__(128) generic_attn_kernel(
    const T* __restrict__ q, const int32_t* __restrict__ q_pos, const T* __restrict__ k,
    const T* __restrict__ v, const int32_t* __restrict__ idx, const float* __restrict__ z_sel,
    int L, int Lq, int Hq, int Hkv, int K, int w, int flags, T* __restrict__ o,
    float* __restrict__ lse) {
  constexpr int EPL = D / 32;
  __shared__ float qsm[4][D];
  const int i = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int G = Hq / Hkv, C = L / S;
  const int p = q_pos ? q_pos[(size_t)b * Lq + i] : i;
  if (ROUTE && is_mask_slot(p)) return;
  if ((flags & RDL_FLAG_CHECKS) && (p < 0 || p >= L)) record_status(RDL_ERR_DEVICE_CHECK);
  const T* kg = k + (size_t)(b * Hkv + g) * L * D;
  const T* vg = v + (size_t)(b * Hkv + g) * L * D;
  for (int hl = warp; hl < G; hl += 4) {
    const int h = g * G + hl;
    const T* qr = q + ((size_t)(b * Lq + i) * Hq + h) * D;
    for (int e = lane; e < D; e += 32) qsm[warp][e] = IO<T>::ld(qr + e);
    __syncwarp();
    float m = -INFINITY, l = 0.f, acc[EPL];
#pragma unroll
    for (int u = 0; u < EPL; ++u) acc[u] = 0.f;
    if (w >= 0) {
      const int j0 = max(0, p - w), j1 = min(L, p + w + 1);
      attend_range<T, D>(qsm[warp], kg, vg, j0, j1, m, l, acc, lane);
    }
    float M = -INFINITY, Zs = 0.f, out[EPL];
#pragma unroll
    for (int u = 0; u < EPL; ++u) out[u] = 0.f;
    // fold one partition part (logit a, normalised vector acc/lpart) into (M, Zs, out)
    auto fold = [&](float a, float lpart, const float* accp) {
      if (a == -INFINITY || lpart <= 0.f) return;
      const float Mn = fmaxf(M, a);
      const float sc = (M == -INFINITY) ? 0.f : expf(M - Mn);
      const float wa = expf(a - Mn);
      Zs = Zs * sc + wa;
#pragma unroll
      for (int u = 0; u < EPL; ++u) out[u] = out[u] * sc + wa * (accp[u] / lpart);
      M = Mn;
    };
    if (l > 0.f) fold(m + logf(l), l, acc);
    if (ROUTE) {
      for (int kk = 0; kk < K; ++kk) {
        const int c = idx[((size_t)(b * Hkv + g) * Lq + i) * K + kk];
        if (c < 0) continue;
        if (c >= C || !chunk_eligible(c, p, w)) {
          if (flags & RDL_FLAG_CHECKS) record_status(RDL_ERR_DEVICE_CHECK);
          if (c >= C) continue;
        }
        float mc = -INFINITY, lc = 0.f, accc[EPL];
#pragma unroll
        for (int u = 0; u < EPL; ++u) accc[u] = 0.f;
        attend_range<T, D>(qsm[warp], kg, vg, c * S, c * S + CONTENT, mc, lc, accc, lane);
        fold(z_sel[((size_t)(b * Hq + h) * Lq + i) * K + kk], lc, accc);
      }
    }
    T* orow = o + ((size_t)(b * Lq + i) * Hq + h) * D;
    const float inv = Zs > 0.f ? 1.f / Zs : 0.f;
#pragma unroll
    for (int u = 0; u < EPL; ++u) IO<T>::st(orow + lane + 32 * u, out[u] * inv);
    if (lse && lane == 0) lse[(size_t)(b * Hq + h) * Lq + i] = Zs > 0.f ? M + logf(Zs) : -INFINITY;
    __syncwarp();
  }
}

// --------------------------------------------------------------------------- mma window
// MODE 0: sliding-window layer output (o bf16, lse).  MODE 1: route-layer local window,
// normalised o_loc (fp32) and its log-sum-exp lambda_loc, consumed by the chunk kernel.
// With nsplit > 1 (few query rows, e.g. decode blocks) the key blocks of a row tile are
// split over blockIdx.z and each split writes its own normalised output and log-sum-exp
// to o_loc / lam_loc plane `split`; the chunk kernel (route) or window_combine_kernel
// (sliding window) merges the planes.
constexpr int WIN_ROWS = 16;
constexpr int WIN_KEYS = 64;

template <int MODE>
__global__ void __launch_bounds__(256) window_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ q_pos,
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v, int L, int Lq,
    int Hq, int Hkv, int w, __nv_bfloat16* __restrict__ o, float* __restrict__ lse,
    float* __restrict__ o_loc, float* __restrict__ lam_loc, int nsplit) {
  constexpr int D = 128;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  unsigned char* Ks = smem_raw;                       // [2][64 rows][256 B]
  unsigned char* Vs = Ks + 2 * WIN_KEYS * 256;        // [2][64][256]
  unsigned char* Qs = Vs + 2 * WIN_KEYS * 256;        // [G][16][256]
  __shared__ int pos_s[WIN_ROWS];
  __shared__ int range_s[2];

  const int G = Hq / Hkv;
  const int bg = blockIdx.y, b = bg / Hkv, g = bg % Hkv;
  const int i0 = blockIdx.x * WIN_ROWS;
  const int tid = threadIdx.x, nthr = blockDim.x;
  const int lane = tid & 31, warp = tid >> 5;
  const int h = g * G + warp;

  if (tid < WIN_ROWS) {
    const int i = i0 + tid;
    pos_s[tid] = (i < Lq) ? (q_pos ? q_pos[(size_t)b * Lq + i] : i) : INT_MIN;
  }
  // Q tile: G heads x 16 rows x 128 (zero rows beyond Lq)
  for (int e = tid; e < G * WIN_ROWS * 16; e += nthr) {
    const int hl = e / (WIN_ROWS * 16), r = (e / 16) % WIN_ROWS, ch = e % 16;
    const int i = min(i0 + r, Lq - 1);
    const __nv_bfloat16* src = q + ((size_t)(b * Lq + i) * Hq + g * G + hl) * D + ch * 8;
    cp_async16(smem_u32(Qs + hl * WIN_ROWS * 256 + swz256(r, ch)), src);
  }
  cp_async_commit();
  __syncthreads();
  if (tid == 0) {
    int pmin = INT_MAX, pmax = INT_MIN;
    for (int r = 0; r < WIN_ROWS; ++r)
      if (pos_s[r] != INT_MIN) { pmin = min(pmin, pos_s[r]); pmax = max(pmax, pos_s[r]); }
    range_s[0] = max(0, pmin - w);
    range_s[1] = min(L, pmax + w + 1);
  }
  __syncthreads();
  const int kbeg = range_s[0], kend = range_s[1];
  const int nblk_all = kend > kbeg ? (kend - kbeg + WIN_KEYS - 1) / WIN_KEYS : 0;
  const int split = blockIdx.z;
  const int per = (nblk_all + nsplit - 1) / nsplit;
  const int blo = min(nblk_all, split * per), bhi = min(nblk_all, blo + per);
  const __nv_bfloat16* kg = k + (size_t)(b * Hkv + g) * L * D;
  const __nv_bfloat16* vg = v + (size_t)(b * Hkv + g) * L * D;

  auto load_block = [&](int blk, int stage) {
    const int base = kbeg + blk * WIN_KEYS;
    for (int e = tid; e < WIN_KEYS * 16; e += nthr) {
      const int r = e / 16, ch = e % 16;
      const int j = min(base + r, L - 1);
      cp_async16(smem_u32(Ks + stage * WIN_KEYS * 256 + swz256(r, ch)), kg + (size_t)j * D + ch * 8);
      cp_async16(smem_u32(Vs + stage * WIN_KEYS * 256 + swz256(r, ch)), vg + (size_t)j * D + ch * 8);
    }
  };
  if (bhi > blo) load_block(blo, 0);
  cp_async_commit();

  const int gq = lane >> 2, tq = lane & 3;
  const bool active = warp < G;
  // per-row state: rows gq and gq + 8 of the tile
  const int pr0 = pos_s[gq], pr1 = pos_s[gq + 8];
  float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
  float oacc[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n) oacc[n][0] = oacc[n][1] = oacc[n][2] = oacc[n][3] = 0.f;
  uint32_t qa[8][4];
  const float sl2 = rsqrtf((float)D) * LOG2E;

  for (int blk = blo; blk < bhi; ++blk) {
    const int stage = (blk - blo) & 1;
    if (blk + 1 < bhi) load_block(blk + 1, stage ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    if (blk == blo && active) {
      const unsigned char* qw = Qs + warp * WIN_ROWS * 256;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        const int r = (lane & 7) + 8 * ((lane >> 3) & 1), ch = 2 * ks + (lane >> 4);
        ldsm_x4(smem_u32(qw + swz256(r, ch)), qa[ks][0], qa[ks][1], qa[ks][2], qa[ks][3]);
      }
    }
    if (active) {
      const unsigned char* kt = Ks + stage * WIN_KEYS * 256;
      const unsigned char* vt = Vs + stage * WIN_KEYS * 256;
      float s[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        s[nt][0] = s[nt][1] = s[nt][2] = s[nt][3] = 0.f;
#pragma unroll
        for (int ks = 0; ks < 8; ks += 2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_u32(kt + swz256(nt * 8 + (lane & 7), 2 * ks + (lane >> 3))), b0, b1, b2, b3);
          mma_bf16(s[nt], qa[ks], b0, b1);
          mma_bf16(s[nt], qa[ks + 1], b2, b3);
        }
      }
      // scale, band mask, online softmax (base 2)
      const int jb = kbeg + blk * WIN_KEYS;
      float bm0 = -INFINITY, bm1 = -INFINITY;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int j = jb + nt * 8 + 2 * tq + e;
          const bool jv = j < kend;
          const bool ok0 = jv && pr0 != INT_MIN && abs(pr0 - j) <= w;
          const bool ok1 = jv && pr1 != INT_MIN && abs(pr1 - j) <= w;
          s[nt][e] = ok0 ? s[nt][e] * sl2 : -INFINITY;
          s[nt][2 + e] = ok1 ? s[nt][2 + e] * sl2 : -INFINITY;
          bm0 = fmaxf(bm0, s[nt][e]);
          bm1 = fmaxf(bm1, s[nt][2 + e]);
        }
      }
      bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, 1));
      bm0 = fmaxf(bm0, __shfl_xor_sync(0xffffffffu, bm0, 2));
      bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, 1));
      bm1 = fmaxf(bm1, __shfl_xor_sync(0xffffffffu, bm1, 2));
      const float mn0 = fmaxf(m0, bm0), mn1 = fmaxf(m1, bm1);
      const float a0 = (mn0 == -INFINITY) ? 1.f : fast_exp2(m0 - mn0);
      const float a1 = (mn1 == -INFINITY) ? 1.f : fast_exp2(m1 - mn1);
      const float ms0 = (mn0 == -INFINITY) ? 0.f : mn0, ms1 = (mn1 == -INFINITY) ? 0.f : mn1;
      float rs0 = 0.f, rs1 = 0.f;
      uint32_t pa[4][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const float p00 = fast_exp2(s[nt][0] - ms0), p01 = fast_exp2(s[nt][1] - ms0);
        const float p10 = fast_exp2(s[nt][2] - ms1), p11 = fast_exp2(s[nt][3] - ms1);
        rs0 += p00 + p01;
        rs1 += p10 + p11;
        const int kk = nt >> 1, hi = nt & 1;
        pa[kk][hi ? 2 : 0] = pack_bf16(p00, p01);
        pa[kk][hi ? 3 : 1] = pack_bf16(p10, p11);
      }
      rs0 += __shfl_xor_sync(0xffffffffu, rs0, 1);
      rs0 += __shfl_xor_sync(0xffffffffu, rs0, 2);
      rs1 += __shfl_xor_sync(0xffffffffu, rs1, 1);
      rs1 += __shfl_xor_sync(0xffffffffu, rs1, 2);
      l0 = l0 * a0 + rs0;
      l1 = l1 * a1 + rs1;
      m0 = mn0;
      m1 = mn1;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        oacc[n][0] *= a0; oacc[n][1] *= a0;
        oacc[n][2] *= a1; oacc[n][3] *= a1;
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
        for (int dn = 0; dn < 16; dn += 2) {
          uint32_t b0, b1, b2, b3;
          const int jj = lane >> 3;
          ldsm_x4_t(smem_u32(vt + swz256(16 * kk + 8 * (jj & 1) + (lane & 7), dn + (jj >> 1))), b0, b1,
                    b2, b3);
          mma_bf16(oacc[dn], pa[kk], b0, b1);
          mma_bf16(oacc[dn + 1], pa[kk], b2, b3);
        }
      }
    }
    __syncthreads();
  }
  cp_async_wait<0>();
  if (!active) return;
  // epilogue: normalise and store (to the split's partial plane when there are splits)
  const bool partial = (MODE == 1) || nsplit > 1;
  const size_t plane = (size_t)gridDim.y / Hkv * Lq * Hq * D, plane_l = (size_t)gridDim.y / Hkv * Hq * Lq;
  float* o_part = o_loc ? o_loc + (size_t)split * plane : nullptr;
  float* l_part = lam_loc ? lam_loc + (size_t)split * plane_l : nullptr;
  const float inv0 = l0 > 0.f ? 1.f / l0 : 0.f, inv1 = l1 > 0.f ? 1.f / l1 : 0.f;
  const float ls0 = l0 > 0.f ? (m0 + __log2f(l0)) * LN2 : -INFINITY;
  const float ls1 = l1 > 0.f ? (m1 + __log2f(l1)) * LN2 : -INFINITY;
#pragma unroll
  for (int half = 0; half < 2; ++half) {
    const int r = gq + 8 * half, i = i0 + r;
    if (i >= Lq) continue;
    const float inv = half ? inv1 : inv0;
    const size_t rowoff = ((size_t)(b * Lq + i) * Hq + h) * D;
#pragma unroll
    for (int dn = 0; dn < 16; ++dn) {
      const int d0 = dn * 8 + 2 * tq;
      const float x0 = oacc[dn][2 * half] * inv, x1 = oacc[dn][2 * half + 1] * inv;
      if (!partial) {
        *reinterpret_cast<uint32_t*>(o + rowoff + d0) = pack_bf16(x0, x1);
      } else {
        *reinterpret_cast<float2*>(o_part + rowoff + d0) = make_float2(x0, x1);
      }
    }
    if (tq == 0) {
      const float ls = half ? ls1 : ls0;
      if (!partial) {
        if (lse) lse[(size_t)(b * Hq + h) * Lq + i] = ls;
      } else {
        l_part[(size_t)(b * Hq + h) * Lq + i] = ls;
      }
    }
  }
}

inline size_t window_mma_smem(int G) { return (size_t)(4 * WIN_KEYS * 256 + G * WIN_ROWS * 256); }

// Sliding-window output from key-split partials: lse = LSE_s lse_s, o = sum_s e^{lse_s-lse} o_s.
// One thread per (row, head, element).
__global__ void window_combine_kernel(const float* __restrict__ o_part, const float* __restrict__ l_part,
                                      int nsplit, int B, int Lq, int Hq, __nv_bfloat16* __restrict__ o,
                                      float* __restrict__ lse) {
  constexpr int D = 128;
  const long long n = (long long)B * Lq * Hq * D;
  const size_t plane = (size_t)n, plane_l = (size_t)B * Hq * Lq;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n; e += (long long)gridDim.x * blockDim.x) {
    const long long rowh = e / D;                 // (b, i, h)
    const int h = (int)(rowh % Hq);
    const long long bi = rowh / Hq;
    const int i = (int)(bi % Lq), b = (int)(bi / Lq);
    const size_t li = (size_t)(b * Hq + h) * Lq + i;
    float mx = -INFINITY;
    for (int s = 0; s < nsplit; ++s) mx = fmaxf(mx, l_part[s * plane_l + li]);
    float z = 0.f, acc = 0.f;
    if (mx != -INFINITY) {
      for (int s = 0; s < nsplit; ++s) {
        const float ls = l_part[s * plane_l + li];
        const float wgt = (ls == -INFINITY) ? 0.f : expf(ls - mx);
        z += wgt;
        acc = fmaf(wgt, o_part[s * plane + e], acc);
      }
    }
    o[e] = __float2bfloat16_rn(z > 0.f ? acc / z : 0.f);
    if (lse && (e % D) == 0) lse[li] = z > 0.f ? mx + logf(z) : -INFINITY;
  }
}

}  // namespace rdl
