// Two-level partition over the selected chunks of the route layer (Prefilling-dLLM v2,
// Figure 3 caption: "Attention mass puts the selected chunk scores and the local-window
// log-sum-exp in one partition, then a second softmax distributes each chunk's mass over
// its content tokens").
//
// Because the chunk logits z_sel and the window's log-sum-exp lambda_loc are known before
// any chunk is read, the partition function Z = e^lambda_loc + sum_c e^{z_c} is fixed up
// front: every part contributes (e^{part logit}/Z) * (its own normalised output), so the
// chunk loop needs no running rescale, and chunk ranges can be split across warps and
// simply summed.
//
// chunk_mma_kernel: one warp per (b, query row, KV group, chunk split).  Per selected
// chunk the warp stages the chunk's K and V (64 x 128 bf16 each) in its own shared
// memory with cp.async (K of the next chunk loads while this chunk's PV runs) and runs
// the product with operands swapped so the GQA group is the MMA N dimension:
//   S^T[64 keys x 8 heads] = K_c[64 x 128] * Q^T[128 x 8]      (m16n8k16, 7 of 8 columns used)
//   O^T[128 x 8]          += V_c^T[128 x 64] * P^T[64 x 8]
// The chunk's mask slot (key 63) is excluded from the second-level softmax.
#pragma once
#include "common.cuh"

namespace rdl {

constexpr int CH_WARPS = 2;                                // warps per CTA
constexpr int CH_WARP_SMEM = 2 * 64 * 256 + 8 * 64 * 2;   // K + V tile + P^T tile

// P^T tile [8 heads][64 keys] bf16, rows of 128 B, 16-byte chunks XOR-swizzled by head.
__device__ __forceinline__ uint32_t swz_pt(int head, int key) {
  return (uint32_t)(head * 128 + ((((key >> 3) ^ head) & 7) << 4) + (key & 7) * 2);
}

__global__ void __launch_bounds__(CH_WARPS * 32) chunk_mma_kernel(
    const __nv_bfloat16* __restrict__ q, const int32_t* __restrict__ q_pos,
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v,
    const int32_t* __restrict__ idx, const float* __restrict__ z_sel,
    const float* __restrict__ o_loc, const float* __restrict__ lam_loc, int L, int Lq, int Hq,
    int Hkv, int K, int w, int nsplit, int flags, __nv_bfloat16* __restrict__ o,
    float* __restrict__ lse, float* __restrict__ o_acc, int nsw) {
  constexpr int D = 128;
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  unsigned char* Kc = smem_raw + warp * CH_WARP_SMEM;
  unsigned char* Vc = Kc + 64 * 256;
  unsigned char* Pt = Vc + 64 * 256;

  const int G = Hq / Hkv, C = L / S;
  long long item = (long long)blockIdx.x * CH_WARPS + warp;
  const int split = (int)(item % nsplit);
  item /= nsplit;
  if (item >= (long long)Lq * Hkv) return;
  const int b = blockIdx.y;
  const int g = (int)(item % Hkv), i = (int)(item / Hkv);
  const int p = q_pos ? q_pos[(size_t)b * Lq + i] : i;
  if (is_mask_slot(p)) return;

  const int gq = lane >> 2, tq = lane & 3;
  const int hA = 2 * tq, hB = 2 * tq + 1;           // heads of this thread's S^T/O^T columns
  const bool vA = hA < G, vB = hB < G;
  // Q^T fragments: column n = gq is head gq of the group
  uint32_t qb[8][2];
  {
    const bool vq = gq < G;
    const __nv_bfloat16* qr = q + ((size_t)(b * Lq + i) * Hq + g * G + (vq ? gq : 0)) * D;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qb[ks][0] = vq ? *reinterpret_cast<const uint32_t*>(qr + 16 * ks + 2 * tq) : 0u;
      qb[ks][1] = vq ? *reinterpret_cast<const uint32_t*>(qr + 16 * ks + 2 * tq + 8) : 0u;
    }
  }
  // fixed partition: M_h = max(lambda_loc, z_h,*), Zs_h = e^{lambda_loc - M} + sum e^{z - M}
  const int32_t* irow = idx + ((size_t)(b * Hkv + g) * Lq + i) * K;
  const size_t zA = ((size_t)(b * Hq + g * G + (vA ? hA : 0)) * Lq + i) * K;
  const size_t zB = ((size_t)(b * Hq + g * G + (vB ? hB : 0)) * Lq + i) * K;
  // window log-sum-exp: merge the key-split planes, lambda = LSE_s lambda_s
  const size_t plane_l = (size_t)gridDim.y * Hq * Lq;
  const size_t liA = (size_t)(b * Hq + g * G + (vA ? hA : 0)) * Lq + i;
  const size_t liB = (size_t)(b * Hq + g * G + (vB ? hB : 0)) * Lq + i;
  float lamA = -INFINITY, lamB = -INFINITY;
  {
    // lanes sharing tq split the window planes (nsw <= 8 * lanes-per-head)
    float la = -INFINITY, lb = -INFINITY, mA = -INFINITY, mB = -INFINITY;
    float lva[2], lvb[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int sw = gq + 8 * u;
      lva[u] = sw < nsw ? lam_loc[sw * plane_l + liA] : -INFINITY;
      lvb[u] = sw < nsw ? lam_loc[sw * plane_l + liB] : -INFINITY;
      mA = fmaxf(mA, lva[u]);
      mB = fmaxf(mB, lvb[u]);
    }
    for (int sw = gq + 16; sw < nsw; sw += 8) {
      mA = fmaxf(mA, lam_loc[sw * plane_l + liA]);
      mB = fmaxf(mB, lam_loc[sw * plane_l + liB]);
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mA = fmaxf(mA, __shfl_xor_sync(0xffffffffu, mA, off));
      mB = fmaxf(mB, __shfl_xor_sync(0xffffffffu, mB, off));
    }
    float sA = 0.f, sB = 0.f;
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      if (lva[u] != -INFINITY) sA += expf(lva[u] - mA);
      if (lvb[u] != -INFINITY) sB += expf(lvb[u] - mB);
    }
    for (int sw = gq + 16; sw < nsw; sw += 8) {
      const float a = lam_loc[sw * plane_l + liA], bb = lam_loc[sw * plane_l + liB];
      if (a != -INFINITY) sA += expf(a - mA);
      if (bb != -INFINITY) sB += expf(bb - mB);
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      sA += __shfl_xor_sync(0xffffffffu, sA, off);
      sB += __shfl_xor_sync(0xffffffffu, sB, off);
    }
    (void)la; (void)lb;
    if (vA && sA > 0.f) lamA = mA + logf(sA);
    if (vB && sB > 0.f) lamB = mB + logf(sB);
  }
  // the 8 lanes sharing tq (same heads) split the K slots: loads in flight together
  float zvA[8], zvB[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int kk = gq + 8 * u;
    zvA[u] = kk < K ? z_sel[zA + kk] : -INFINITY;
    zvB[u] = kk < K ? z_sel[zB + kk] : -INFINITY;
  }
  float MA = lamA, MB = lamB;
#pragma unroll
  for (int u = 0; u < 8; ++u) { MA = fmaxf(MA, zvA[u]); MB = fmaxf(MB, zvB[u]); }
  for (int kk = gq + 64; kk < K; kk += 8) { MA = fmaxf(MA, z_sel[zA + kk]); MB = fmaxf(MB, z_sel[zB + kk]); }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    MA = fmaxf(MA, __shfl_xor_sync(0xffffffffu, MA, off));
    MB = fmaxf(MB, __shfl_xor_sync(0xffffffffu, MB, off));
  }
  if (MA == -INFINITY) MA = 0.f;   // no part at all (cannot happen for valid selections)
  if (MB == -INFINITY) MB = 0.f;
  float ZA = 0.f, ZB = 0.f;
#pragma unroll
  for (int u = 0; u < 8; ++u) { ZA += expf(zvA[u] - MA); ZB += expf(zvB[u] - MB); }
  for (int kk = gq + 64; kk < K; kk += 8) { ZA += expf(z_sel[zA + kk] - MA); ZB += expf(z_sel[zB + kk] - MB); }
#pragma unroll
  for (int off = 4; off < 32; off <<= 1) {
    ZA += __shfl_xor_sync(0xffffffffu, ZA, off);
    ZB += __shfl_xor_sync(0xffffffffu, ZB, off);
  }
  ZA += (lamA == -INFINITY) ? 0.f : expf(lamA - MA);
  ZB += (lamB == -INFINITY) ? 0.f : expf(lamB - MB);
  const float invZA = ZA > 0.f ? 1.f / ZA : 0.f, invZB = ZB > 0.f ? 1.f / ZB : 0.f;

  const int per = (K + nsplit - 1) / nsplit;
  const int k_lo = split * per, k_hi = min(K, k_lo + per);
  const __nv_bfloat16* kg = k + (size_t)(b * Hkv + g) * L * D;
  const __nv_bfloat16* vg = v + (size_t)(b * Hkv + g) * L * D;

  auto chunk_at = [&](int kk) -> int {
    if (kk >= k_hi) return -1;
    int c = irow[kk];
    if (c >= 0 && (c >= C || !chunk_eligible(c, p, w))) {
      if (flags & RDL_FLAG_CHECKS) record_status(RDL_ERR_DEVICE_CHECK);
      if (c >= C) c = -1;
    }
    return c;
  };
  auto load_tile = [&](unsigned char* dst, const __nv_bfloat16* src_base, int c) {
    const __nv_bfloat16* src = src_base + (size_t)c * S * D;
#pragma unroll
    for (int u = 0; u < 32; ++u) {              // 64 rows x 16 chunks / 32 lanes
      const int e = u * 32 + lane, r = e >> 4, ch = e & 15;
      cp_async16(smem_u32(dst + swz256(r, ch)), src + (size_t)r * D + ch * 8);
    }
  };

  float oacc[8][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt) oacc[mt][0] = oacc[mt][1] = oacc[mt][2] = oacc[mt][3] = 0.f;
  const float sl2 = rsqrtf((float)D) * LOG2E;

  int kk = k_lo;
  int c = chunk_at(kk);
  while (kk < k_hi && c < 0 && irow[kk] >= 0) c = chunk_at(++kk);   // skip invalid (checks)
  if (c >= 0) { load_tile(Kc, kg, c); }
  cp_async_commit();
  if (c >= 0) { load_tile(Vc, vg, c); }
  cp_async_commit();

  while (kk < k_hi && c >= 0) {
    // ---- S^T = K_c Q^T
    cp_async_wait<1>();
    __syncwarp();
    float s[4][4];
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
      s[mt][0] = s[mt][1] = s[mt][2] = s[mt][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        uint32_t a[4];
        const int r = mt * 16 + (lane & 7) + 8 * ((lane >> 3) & 1), ch = 2 * ks + (lane >> 4);
        ldsm_x4(smem_u32(Kc + swz256(r, ch)), a[0], a[1], a[2], a[3]);
        mma_bf16(s[mt], a, qb[ks][0], qb[ks][1]);
      }
    }
    __syncwarp();
    // next chunk's K streams in while this chunk's softmax and PV run
    int kn = kk + 1;
    int cn = chunk_at(kn);
    while (kn < k_hi && cn < 0 && irow[kn] >= 0) cn = chunk_at(++kn);
    if (cn >= 0) load_tile(Kc, kg, cn);
    cp_async_commit();
    // ---- second-level softmax over the 63 content keys, per head (column)
    float mxA = -INFINITY, mxB = -INFINITY;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int key = mt * 16 + gq + 8 * hr;
        const bool kv = key < CONTENT;
        s[mt][2 * hr] = kv ? s[mt][2 * hr] * sl2 : -INFINITY;
        s[mt][2 * hr + 1] = kv ? s[mt][2 * hr + 1] * sl2 : -INFINITY;
        mxA = fmaxf(mxA, s[mt][2 * hr]);
        mxB = fmaxf(mxB, s[mt][2 * hr + 1]);
      }
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      mxA = fmaxf(mxA, __shfl_xor_sync(0xffffffffu, mxA, off));
      mxB = fmaxf(mxB, __shfl_xor_sync(0xffffffffu, mxB, off));
    }
    float smA = 0.f, smB = 0.f;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        s[mt][2 * hr] = fast_exp2(s[mt][2 * hr] - mxA);
        s[mt][2 * hr + 1] = fast_exp2(s[mt][2 * hr + 1] - mxB);
        smA += s[mt][2 * hr];
        smB += s[mt][2 * hr + 1];
      }
    }
#pragma unroll
    for (int off = 4; off < 32; off <<= 1) {
      smA += __shfl_xor_sync(0xffffffffu, smA, off);
      smB += __shfl_xor_sync(0xffffffffu, smB, off);
    }
    // chunk mass e^{z_c - M}/Zs spread by the chunk's own softmax
    const float fA = vA ? expf(z_sel[zA + kk] - MA) * invZA / smA : 0.f;
    const float fB = vB ? expf(z_sel[zB + kk] - MB) * invZB / smB : 0.f;
#pragma unroll
    for (int mt = 0; mt < 4; ++mt) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int key = mt * 16 + gq + 8 * hr;
        *reinterpret_cast<__nv_bfloat16*>(Pt + swz_pt(hA, key)) = __float2bfloat16_rn(s[mt][2 * hr] * fA);
        *reinterpret_cast<__nv_bfloat16*>(Pt + swz_pt(hB, key)) = __float2bfloat16_rn(s[mt][2 * hr + 1] * fB);
      }
    }
    __syncwarp();
    uint32_t pb[4][2];
#pragma unroll
    for (int kp = 0; kp < 4; kp += 2) {
      const int jj = lane >> 3;
      ldsm_x4(smem_u32(Pt + swz_pt(lane & 7, (2 * kp + jj) * 8)), pb[kp][0], pb[kp][1],
              pb[kp + 1][0], pb[kp + 1][1]);
    }
    // ---- O^T += V_c^T P^T
    cp_async_wait<1>();
    __syncwarp();
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
      for (int k2 = 0; k2 < 4; ++k2) {
        uint32_t a[4];
        const int jj = lane >> 3;
        ldsm_x4_t(smem_u32(Vc + swz256(16 * k2 + 8 * (jj >> 1) + (lane & 7), 2 * mt + (jj & 1))), a[0],
                  a[1], a[2], a[3]);
        mma_bf16(oacc[mt], a, pb[k2][0], pb[k2][1]);
      }
    }
    __syncwarp();
    if (cn >= 0) load_tile(Vc, vg, cn);
    cp_async_commit();
    kk = kn;
    c = cn;
  }
  cp_async_wait<0>();
  __syncwarp();

  // ---- local window part (one split adds it)
  if (split == 0) {
    // each key-split plane of the window enters with mass e^{lambda_s - M}/Zs
    const size_t plane = (size_t)gridDim.y * Lq * Hq * D;
    for (int sw = 0; sw < nsw; ++sw) {
      const float lsA = vA ? lam_loc[sw * plane_l + liA] : -INFINITY;
      const float lsB = vB ? lam_loc[sw * plane_l + liB] : -INFINITY;
      const float wA = (lsA != -INFINITY) ? expf(lsA - MA) * invZA : 0.f;
      const float wB = (lsB != -INFINITY) ? expf(lsB - MB) * invZB : 0.f;
      const float* olA = o_loc + sw * plane + ((size_t)(b * Lq + i) * Hq + g * G + (vA ? hA : 0)) * D;
      const float* olB = o_loc + sw * plane + ((size_t)(b * Lq + i) * Hq + g * G + (vB ? hB : 0)) * D;
#pragma unroll
      for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
        for (int hr = 0; hr < 2; ++hr) {
          const int dd = mt * 16 + gq + 8 * hr;
          if (wA != 0.f) oacc[mt][2 * hr] += wA * olA[dd];
          if (wB != 0.f) oacc[mt][2 * hr + 1] += wB * olB[dd];
        }
      }
    }
    if (lse && gq == 0) {
      if (vA) lse[(size_t)(b * Hq + g * G + hA) * Lq + i] = MA + logf(ZA);
      if (vB) lse[(size_t)(b * Hq + g * G + hB) * Lq + i] = MB + logf(ZB);
    }
  }
  if (nsplit == 1) {
    // stage O as bf16 [8 heads][128] in the K tile, then write 16-byte rows
    __nv_bfloat16* Os = reinterpret_cast<__nv_bfloat16*>(Kc);
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int dd = mt * 16 + gq + 8 * hr;
        Os[hA * D + dd] = __float2bfloat16_rn(oacc[mt][2 * hr]);
        Os[hB * D + dd] = __float2bfloat16_rn(oacc[mt][2 * hr + 1]);
      }
    }
    __syncwarp();
    __nv_bfloat16* orow = o + ((size_t)(b * Lq + i) * Hq + g * G) * D;
    for (int e = lane; e < G * 16; e += 32) {
      const int hh = e >> 4, ch = e & 15;
      *reinterpret_cast<uint4*>(orow + hh * D + ch * 8) =
          *reinterpret_cast<const uint4*>(Os + hh * D + ch * 8);
    }
  } else {
    // this split's partial; the finalize kernel sums the splits in a fixed order
    const size_t plane = (size_t)gridDim.y * Lq * Hq * D;
    float* arow = o_acc + (size_t)split * plane + ((size_t)(b * Lq + i) * Hq + g * G) * D;
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int dd = mt * 16 + gq + 8 * hr;
        if (vA) arow[hA * D + dd] = oacc[mt][2 * hr];
        if (vB) arow[hB * D + dd] = oacc[mt][2 * hr + 1];
      }
    }
  }
}

// Split mode: o (bf16) of the content rows = sum of the splits' partials, in split order
// (deterministic: no atomics).
__global__ void chunk_finalize_kernel(const float* __restrict__ o_acc, int nsplit,
                                      const int32_t* __restrict__ q_pos, int Lq, int HqD, int B,
                                      __nv_bfloat16* __restrict__ o) {
  const long long n = (long long)B * Lq * HqD;
  for (long long e = (long long)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (long long)gridDim.x * blockDim.x) {
    const long long row = e / HqD;
    const int b = (int)(row / Lq), i = (int)(row % Lq);
    const int p = q_pos ? q_pos[(size_t)b * Lq + i] : i;
    if (is_mask_slot(p)) continue;
    float acc = 0.f;
    for (int s = 0; s < nsplit; ++s) acc += o_acc[(size_t)s * n + e];
    o[e] = __float2bfloat16_rn(acc);
  }
}

}  // namespace rdl
