// Summary pooling: summary key s_c, pooling entropy H_c and the mask slot's own output
// (Prefilling-dLLM v2, Figure 3 caption: the mask's query pools the chunk's content keys
// with an intra-chunk softmax; the weighted sum is the summary key; the entropy of the
// pooling weights is the second routing signal).
//
// One CTA per (chunk c, KV head g, batch b): the chunk's 63 content keys (and values)
// are read from HBM once into shared memory and reused by every query head of the group.
// The pass streams K/V once, so it is HBM-bound.  Three forms: bf16 with d = 128 and at most
// 8 heads per group takes summary_pool_mma_kernel (tensor cores, K/V slabs by TMA); other
// bf16 shapes take summary_pool_bulk_kernel (one bulk copy per slab, bf16 in shared memory);
// fp32 inputs, or mask-query strides that do not keep a lane's elements aligned, take
// summary_pool_kernel (fp32 staging).
#pragma once
#include <type_traits>
#include "common.cuh"
#include "tc.cuh"
#include "tmap.cuh"

namespace rdl {

template <typename T, int D>
__global__ void __launch_bounds__(256) summary_pool_kernel(
    const T* __restrict__ q_mask, long long q_chunk_stride, long long q_batch_stride,
    const T* __restrict__ k, const T* __restrict__ v, int L, int Hq, int Hkv, int flags,
    float* __restrict__ summary, float* __restrict__ entropy, T* __restrict__ o_mask) {
  constexpr int DP = D + 1;                 // padded fp32 row: lane-per-key reads conflict-free
  extern __shared__ float smem[];
  float* Ks = smem;                         // [63][DP]
  float* Vs = Ks + CONTENT * DP;            // [63][DP] (only when v)
  float* Qs = Vs + (v ? CONTENT * DP : 0);  // [8 warps][D]

  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int C = L / S, G = Hq / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t kv_base = ((size_t)(b * Hkv + g) * L + (size_t)c * S) * D;

  // stage content keys / values (8 elements per thread-step)
  constexpr int V8 = D / 8;
  for (int e = tid; e < CONTENT * V8; e += blockDim.x) {
    const int row = e / V8, col = (e % V8) * 8;
    float f[8];
    load8(k + kv_base + (size_t)row * D + col, f);
#pragma unroll
    for (int u = 0; u < 8; ++u) Ks[row * DP + col + u] = f[u];
    if (v) {
      load8(v + kv_base + (size_t)row * D + col, f);
#pragma unroll
      for (int u = 0; u < 8; ++u) Vs[row * DP + col + u] = f[u];
    }
  }
  __syncthreads();

  const float tau = rsqrtf((float)D);
  const bool mean = (flags & RDL_FLAG_MEAN_SUMMARY) != 0;
  float* qs = Qs + warp * D;
  for (int hl = warp; hl < G; hl += blockDim.x / 32) {
    const int h = g * G + hl;
    const T* qrow = q_mask + (size_t)b * q_batch_stride + (size_t)c * q_chunk_stride + (size_t)h * D;
    for (int e = lane; e < D; e += 32) qs[e] = IO<T>::ld(qrow + e);
    __syncwarp();
    // lane j owns keys j and j + 32 (the latter only for j < 31)
    float l0 = 0.f, l1 = 0.f;
    const bool has1 = lane + 32 < CONTENT;
    if (!mean) {
      const float* k0 = Ks + lane * DP;
      const float* k1 = Ks + (has1 ? lane + 32 : lane) * DP;
#pragma unroll 8
      for (int e = 0; e < D; ++e) {
        const float qe = qs[e];
        l0 = fmaf(qe, k0[e], l0);
        l1 = fmaf(qe, k1[e], l1);
      }
      l0 *= tau;
      l1 = has1 ? l1 * tau : -INFINITY;
    } else {
      l1 = has1 ? 0.f : -INFINITY;
    }
    const float m = warp_max(fmaxf(l0, l1));
    const float e0 = expf(l0 - m), e1 = has1 ? expf(l1 - m) : 0.f;
    const float z = warp_sum(e0 + e1);
    const float inv = 1.f / z;
    const float a0 = e0 * inv, a1 = e1 * inv;
    // H = -sum a ln a = ln Z - sum a (l - m)
    const float sal = warp_sum(a0 * (l0 - m) + (has1 ? a1 * (l1 - m) : 0.f));
    const float H = logf(z) - sal;

    // weighted sums: lane owns elements e = lane + 32 u
    constexpr int EPL = D / 32;
    float sacc[EPL], oacc[EPL];
#pragma unroll
    for (int u = 0; u < EPL; ++u) sacc[u] = oacc[u] = 0.f;
    for (int j = 0; j < CONTENT; ++j) {
      const float aj = __shfl_sync(0xffffffffu, j < 32 ? a0 : a1, j & 31);
#pragma unroll
      for (int u = 0; u < EPL; ++u) {
        sacc[u] = fmaf(aj, Ks[j * DP + lane + 32 * u], sacc[u]);
        if (v) oacc[u] = fmaf(aj, Vs[j * DP + lane + 32 * u], oacc[u]);
      }
    }
    float* srow = summary + ((size_t)(b * Hq + h) * C + c) * D;
    if (flags & RDL_FLAG_SPLIT_SUMMARY) {
      // the same 4D bytes as D bf16 hi terms, then D bf16 lo terms (s = hi + lo)
      __nv_bfloat16* hrow = reinterpret_cast<__nv_bfloat16*>(srow);
#pragma unroll
      for (int u = 0; u < EPL; ++u) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(sacc[u]);
        hrow[lane + 32 * u] = hi;
        hrow[D + lane + 32 * u] = __float2bfloat16_rn(sacc[u] - __bfloat162float(hi));
      }
    } else {
#pragma unroll
      for (int u = 0; u < EPL; ++u) srow[lane + 32 * u] = sacc[u];
    }
    if (lane == 0) entropy[(size_t)(b * Hq + h) * C + c] = H;
    if (o_mask && v) {
      T* orow = o_mask + (size_t)b * q_batch_stride + (size_t)c * q_chunk_stride + (size_t)h * D;
#pragma unroll
      for (int u = 0; u < EPL; ++u) IO<T>::st(orow + lane + 32 * u, oacc[u]);
    }
    __syncwarp();
  }
}

// E consecutive bf16 values (E = 2 or 4, 4- or 8-byte aligned) to / from fp32
template <int E>
__device__ __forceinline__ void ld_bf16_vec(const __nv_bfloat16* p, float* f) {
  static_assert(E == 2 || E == 4, "two or four elements");
  if constexpr (E == 4) {
    const uint2 r = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.x));
    const float2 c = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&r.y));
    f[0] = a.x; f[1] = a.y; f[2] = c.x; f[3] = c.y;
  } else {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
    f[0] = a.x; f[1] = a.y;
  }
}
template <int E>
__device__ __forceinline__ void st_bf16_vec(__nv_bfloat16* p, const float* f) {
  static_assert(E == 2 || E == 4, "two or four elements");
  const __nv_bfloat162 a = __floats2bfloat162_rn(f[0], f[1]);
  if constexpr (E == 4) {
    const __nv_bfloat162 c = __floats2bfloat162_rn(f[2], f[3]);
    uint2 r;
    r.x = *reinterpret_cast<const uint32_t*>(&a);
    r.y = *reinterpret_cast<const uint32_t*>(&c);
    *reinterpret_cast<uint2*>(p) = r;
  } else {
    *reinterpret_cast<__nv_bfloat162*>(p) = a;
  }
}
// One halving exchange of the reduce-scatter: p[0 .. 2 DIST) -> p[0 .. DIST), keeping the
// half whose key bit DIST equals the lane's bit DIST and adding the partner's share of it.
template <int DIST>
__device__ __forceinline__ void rs_step(float* p, int lane) {
  const bool upper = (lane & DIST) != 0;
#pragma unroll
  for (int t = 0; t < DIST; ++t) {
    const float send = upper ? p[t] : p[DIST + t];
    const float keep = upper ? p[DIST + t] : p[t];
    p[t] = keep + __shfl_xor_sync(0xffffffffu, send, DIST);
  }
}

// bf16 inputs: the chunk's 63 content keys (and values) arrive in shared memory by one bulk
// copy each (16128 contiguous bytes of the [B, Hkv, L, d] cache) and stay bf16, so a CTA
// holds 32 KB and several CTAs share an SM with their copies in flight at once.  Warp hl
// takes head hl of the group; lane l owns the E = d/32 consecutive elements [E l, E l + E)
// of every row (conflict-free row reads).  The 63 logits: per 32-key half, every lane forms
// its partial dot products with its E elements, and a reduce-scatter over the warp (halving
// exchanges at lane distances 16, 8, 4, 2, 1) leaves lane l the full logit of key l of the
// half.  Softmax, entropy and the weighted sums then follow as in the fp32 kernel above.
template <int D>
__global__ void __launch_bounds__(256) summary_pool_bulk_kernel(
    const __nv_bfloat16* __restrict__ q_mask, long long q_chunk_stride, long long q_batch_stride,
    const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v, int L, int Hq, int Hkv,
    int flags, float* __restrict__ summary, float* __restrict__ entropy, __nv_bfloat16* __restrict__ o_mask) {
  constexpr int E = D / 32;                       // elements per lane
  constexpr unsigned ROW_BYTES = CONTENT * D * 2;  // one slab of content rows (multiple of 16)
  extern __shared__ __align__(128) unsigned char sp_raw[];
  __nv_bfloat16* Ks = reinterpret_cast<__nv_bfloat16*>(sp_raw);
  __nv_bfloat16* Vs = Ks + CONTENT * D;
  __shared__ __align__(8) uint64_t bar;

  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int C = L / S, G = Hq / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const size_t kv_base = ((size_t)(b * Hkv + g) * L + (size_t)c * S) * D;
  if (tid == 0) {
    tc::mbar_init(&bar, 1);
    tc::mbar_fence_init();
    tc::mbar_arrive_expect_tx(&bar, v ? 2 * ROW_BYTES : ROW_BYTES);
    tc::bulk_load(Ks, k + kv_base, ROW_BYTES, &bar);
    if (v) tc::bulk_load(Vs, v + kv_base, ROW_BYTES, &bar);
  }
  __syncthreads();

  const float tau = rsqrtf((float)D);
  const bool mean = (flags & RDL_FLAG_MEAN_SUMMARY) != 0;
  const bool has1 = lane + 32 < CONTENT;
  bool landed = false;
  for (int hl = warp; hl < G; hl += blockDim.x / 32) {
    const int h = g * G + hl;
    const __nv_bfloat16* qrow = q_mask + (size_t)b * q_batch_stride + (size_t)c * q_chunk_stride + (size_t)h * D;
    float qv[E];
    ld_bf16_vec<E>(qrow + E * lane, qv);
    if (!landed) {
      if (!__all_sync(0xffffffffu, tc::mbar_wait(&bar, 0))) return;   // bounded; status recorded
      landed = true;
    }
    float l0 = 0.f, l1 = 0.f;
    if (!mean) {
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        float p[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const int key = 32 * half + j;
          float acc = 0.f;
          if (key < CONTENT) {
            float kv[E];
            ld_bf16_vec<E>(Ks + key * D + E * lane, kv);
#pragma unroll
            for (int e = 0; e < E; ++e) acc = fmaf(qv[e], kv[e], acc);
          }
          p[j] = acc;
        }
        // reduce-scatter: after the exchange at distance s a lane keeps the values whose key
        // bit s equals its own lane bit s; at the end lane l holds key l of the half
        rs_step<16>(p, lane);
        rs_step<8>(p, lane);
        rs_step<4>(p, lane);
        rs_step<2>(p, lane);
        rs_step<1>(p, lane);
        if (half == 0) l0 = p[0] * tau; else l1 = p[0] * tau;
      }
      if (!has1) l1 = -INFINITY;
    } else {
      l1 = has1 ? 0.f : -INFINITY;
    }
    const float m = warp_max(fmaxf(l0, l1));
    const float e0 = expf(l0 - m), e1 = has1 ? expf(l1 - m) : 0.f;
    const float z = warp_sum(e0 + e1);
    const float inv = 1.f / z;
    const float a0 = e0 * inv, a1 = e1 * inv;
    const float sal = warp_sum(a0 * (l0 - m) + (has1 ? a1 * (l1 - m) : 0.f));
    const float H = logf(z) - sal;

    float sacc[E], oacc[E];
#pragma unroll
    for (int e = 0; e < E; ++e) sacc[e] = oacc[e] = 0.f;
#pragma unroll 4
    for (int j = 0; j < CONTENT; ++j) {
      const float aj = __shfl_sync(0xffffffffu, j < 32 ? a0 : a1, j & 31);
      float kv[E];
      ld_bf16_vec<E>(Ks + j * D + E * lane, kv);
#pragma unroll
      for (int e = 0; e < E; ++e) sacc[e] = fmaf(aj, kv[e], sacc[e]);
      if (v) {
        ld_bf16_vec<E>(Vs + j * D + E * lane, kv);
#pragma unroll
        for (int e = 0; e < E; ++e) oacc[e] = fmaf(aj, kv[e], oacc[e]);
      }
    }
    float* srow = summary + ((size_t)(b * Hq + h) * C + c) * D;
    if (flags & RDL_FLAG_SPLIT_SUMMARY) {
      // the same 4D bytes as D bf16 hi terms, then D bf16 lo terms (s = hi + lo)
      __nv_bfloat16* hrow = reinterpret_cast<__nv_bfloat16*>(srow);
      float hv[E], lv[E];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const __nv_bfloat16 hi = __float2bfloat16_rn(sacc[e]);
        hv[e] = __bfloat162float(hi);
        lv[e] = sacc[e] - hv[e];
      }
      st_bf16_vec<E>(hrow + E * lane, hv);
      st_bf16_vec<E>(hrow + D + E * lane, lv);
    } else {
#pragma unroll
      for (int e = 0; e < E; ++e) srow[E * lane + e] = sacc[e];
    }
    if (lane == 0) entropy[(size_t)(b * Hq + h) * C + c] = H;
    if (o_mask && v) {
      __nv_bfloat16* orow = o_mask + (size_t)b * q_batch_stride + (size_t)c * q_chunk_stride + (size_t)h * D;
      st_bf16_vec<E>(orow + E * lane, oacc);
    }
  }
}

// bf16, d = 128: the same pooling on tensor cores (mma.sync, fp32 accumulate).  The chunk's K
// and V slabs arrive by TMA with the 128-byte swizzle (conflict-free ldmatrix); the group's
// mask queries are the A operand (rows = head slots 0-7, rows 8-15 zero):
//     logits  L = Q_mask K^T          (16 x 64, exact bf16 products, fp32 sums)
//     softmax over the 63 content keys per head (quad shuffles), entropy as above
//     s = a K, o = a V                (a split into bf16 hi + lo terms: s to ~2^-17)
// CTA = (chunk, KV head, batch), 4 warps: every warp forms the logits and the softmax of all
// heads (cheap), then the weighted sums for its quarter of the head dimensions.
constexpr int SPM_THREADS = 128;
__device__ __forceinline__ uint32_t spm_kv_off(int row, int col) {   // [2 halves][64 rows][128 B]
  return (uint32_t)((col >> 6) * 8192 + row * 128 + ((((col & 63) >> 3) ^ (row & 7)) << 4) + (col & 7) * 2);
}
__global__ void __launch_bounds__(SPM_THREADS) summary_pool_mma_kernel(
    const __grid_constant__ CUtensorMap kmap, const __grid_constant__ CUtensorMap vmap,
    const __nv_bfloat16* __restrict__ q_mask, long long q_chunk_stride, long long q_batch_stride, int with_v,
    int L, int Hq, int Hkv, int flags, float* __restrict__ summary, float* __restrict__ entropy,
    __nv_bfloat16* __restrict__ o_mask) {
  constexpr int D = 128;
  extern __shared__ unsigned char spm_raw[];
  unsigned char* sm = spm_raw + ((1024u - (smem_u32(spm_raw) & 1023u)) & 1023u);
  __shared__ __align__(8) uint64_t bar;
  const int c = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int C = L / S, G = Hq / Hkv;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gq = lane >> 2, tq = lane & 3;
  if (tid == 0) {
    tc::mbar_init(&bar, 1);
    tc::mbar_fence_init();
    const int row0 = (b * Hkv + g) * L + c * S;
    tc::mbar_arrive_expect_tx(&bar, with_v ? 32768u : 16384u);
    tc::tma_load_3d(sm, &kmap, 0, row0, 0, &bar);
    if (with_v) tc::tma_load_3d(sm + 16384, &vmap, 0, row0, 0, &bar);
  }
  // A fragments of the mask queries (head slot gq; rows 8-15 of the tile are zero)
  uint32_t qa[8][2];
  {
    const bool on = gq < G;
    const __nv_bfloat16* qrow = q_mask + (size_t)b * q_batch_stride + (size_t)c * q_chunk_stride + (size_t)(g * G + (on ? gq : 0)) * D;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      qa[ks][0] = on ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * tq) : 0u;
      qa[ks][1] = on ? *reinterpret_cast<const uint32_t*>(qrow + 16 * ks + 2 * tq + 8) : 0u;
    }
  }
  __syncthreads();
  if (!tc::mbar_wait(&bar, 0)) return;   // bounded; status recorded
  const uint32_t kst = smem_u32(sm), vst = kst + 16384;
  const float tau = rsqrtf((float)D);
  const bool mean = (flags & RDL_FLAG_MEAN_SUMMARY) != 0;
  // ---- logits (row gq: head slot gq; columns 8 nt + 2 tq + {0, 1}: keys)
  float sc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
  if (!mean) {
    const int mi = lane >> 3;
#pragma unroll
    for (int ks = 0; ks < 8; ++ks) {
      const uint32_t a[4] = {qa[ks][0], 0u, qa[ks][1], 0u};
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t b0, b1, b2, b3;
        const int key = 16 * np + 8 * (mi >> 1) + (lane & 7), col = 16 * ks + 8 * (mi & 1);
        ldsm_x4(kst + spm_kv_off(key, col), b0, b1, b2, b3);
        mma_bf16(sc[2 * np], a, b0, b1);
        mma_bf16(sc[2 * np + 1], a, b2, b3);
      }
    }
  }
  // ---- softmax over the 63 content keys of head slot gq (key 63 is the mask slot)
  float l[16];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int key = 8 * nt + 2 * tq + e;
      l[2 * nt + e] = key < CONTENT ? sc[nt][e] * tau : -INFINITY;
    }
  float m = l[0];
#pragma unroll
  for (int x = 1; x < 16; ++x) m = fmaxf(m, l[x]);
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
  m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
  float ex[16], z = 0.f;
#pragma unroll
  for (int x = 0; x < 16; ++x) {
    ex[x] = l[x] == -INFINITY ? 0.f : expf(l[x] - m);
    z += ex[x];
  }
  z += __shfl_xor_sync(0xffffffffu, z, 1);
  z += __shfl_xor_sync(0xffffffffu, z, 2);
  const float inv = 1.f / z;
  float sal = 0.f;
#pragma unroll
  for (int x = 0; x < 16; ++x) {
    ex[x] *= inv;                                   // pooling weight a_j
    if (l[x] != -INFINITY) sal += ex[x] * (l[x] - m);
  }
  sal += __shfl_xor_sync(0xffffffffu, sal, 1);
  sal += __shfl_xor_sync(0xffffffffu, sal, 2);
  const float H = logf(z) - sal;
  // ---- A fragments of the weights (split bf16 hi + lo), FA2 layout of the logit tiles
  uint32_t ph[4][4], pl[4][4];
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const float a0 = ex[2 * (2 * kk + half)], a1 = ex[2 * (2 * kk + half) + 1];
      const __nv_bfloat16 h0 = __float2bfloat16_rn(a0), h1 = __float2bfloat16_rn(a1);
      ph[kk][2 * half] = pack_bf16(__bfloat162float(h0), __bfloat162float(h1));
      pl[kk][2 * half] = pack_bf16(a0 - __bfloat162float(h0), a1 - __bfloat162float(h1));
      ph[kk][2 * half + 1] = 0u;                    // rows 8-15
      pl[kk][2 * half + 1] = 0u;
    }
  }
  // ---- s = a K and o = a V for head dims [32 warp, 32 warp + 32)
  float sacc[4][4], oacc[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) sacc[nt][e] = oacc[nt][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {
    const int mi = lane >> 3;
#pragma unroll
    for (int mm = 0; mm < 2; ++mm) {
      const int key = 16 * kk + 8 * (mi & 1) + (lane & 7), col = 32 * warp + 16 * mm + 8 * (mi >> 1);
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(kst + spm_kv_off(key, col), b0, b1, b2, b3);
      mma_bf16(sacc[2 * mm], ph[kk], b0, b1);
      mma_bf16(sacc[2 * mm], pl[kk], b0, b1);
      mma_bf16(sacc[2 * mm + 1], ph[kk], b2, b3);
      mma_bf16(sacc[2 * mm + 1], pl[kk], b2, b3);
      if (with_v) {
        ldsm_x4_t(vst + spm_kv_off(key, col), b0, b1, b2, b3);
        mma_bf16(oacc[2 * mm], ph[kk], b0, b1);
        mma_bf16(oacc[2 * mm], pl[kk], b0, b1);
        mma_bf16(oacc[2 * mm + 1], ph[kk], b2, b3);
        mma_bf16(oacc[2 * mm + 1], pl[kk], b2, b3);
      }
    }
  }
  if (gq >= G) return;
  const int h = g * G + gq;
  float* srow = summary + ((size_t)(b * Hq + h) * C + c) * D;
#pragma unroll
  for (int nt = 0; nt < 4; ++nt) {
    const int col = 32 * warp + 8 * nt + 2 * tq;
    if (flags & RDL_FLAG_SPLIT_SUMMARY) {
      // the same 4D bytes as D bf16 hi terms, then D bf16 lo terms (s = hi + lo)
      __nv_bfloat16* hrow = reinterpret_cast<__nv_bfloat16*>(srow);
      const __nv_bfloat16 h0 = __float2bfloat16_rn(sacc[nt][0]), h1 = __float2bfloat16_rn(sacc[nt][1]);
      *reinterpret_cast<uint32_t*>(hrow + col) = pack_bf16(__bfloat162float(h0), __bfloat162float(h1));
      *reinterpret_cast<uint32_t*>(hrow + D + col) =
          pack_bf16(sacc[nt][0] - __bfloat162float(h0), sacc[nt][1] - __bfloat162float(h1));
    } else {
      *reinterpret_cast<float2*>(srow + col) = make_float2(sacc[nt][0], sacc[nt][1]);
    }
    if (with_v) {
      __nv_bfloat16* orow = o_mask + (size_t)b * q_batch_stride + (size_t)c * q_chunk_stride + (size_t)h * D;
      *reinterpret_cast<uint32_t*>(orow + col) = pack_bf16(oacc[nt][0], oacc[nt][1]);
    }
  }
  if (warp == 0 && tq == 0) entropy[(size_t)(b * Hq + h) * C + c] = H;
}

template <typename T, int D>
cudaError_t launch_summary_pool(const void* q_mask, long long qcs, long long qbs, const void* k,
                                const void* v, const rdl_dims& dm, float* summary, float* entropy,
                                void* o_mask, cudaStream_t st) {
  const int C = dm.L / S;
  const bool with_v = v != nullptr && o_mask != nullptr;
  // the bulk kernel reads and writes a lane's D/32 mask-query elements as one vector: the
  // strides must keep every mask row aligned to it
  constexpr long long kVec = D / 32;
  if (std::is_same<T, __nv_bfloat16>::value && D == 128 && dm.Hq / dm.Hkv <= 8 && qcs % 2 == 0 && qbs % 2 == 0) {
    // tensor-core pooling (the mask-query rows are read as bf16 pairs)
    CUtensorMap kmap, vmap;
    const unsigned long long rows = (unsigned long long)dm.B * dm.Hkv * dm.L;
    if (!make_tmap_kv_halves(&kmap, k, rows) || (with_v && !make_tmap_kv_halves(&vmap, v, rows)))
      return cudaErrorInvalidValue;
    if (!with_v) vmap = kmap;
    const size_t smem = 32768 + 1024;
    cudaError_t e = cudaFuncSetAttribute(summary_pool_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(C, dm.Hkv, dm.B);
    count_launch();
    summary_pool_mma_kernel<<<grid, SPM_THREADS, smem, st>>>(
        kmap, vmap, static_cast<const __nv_bfloat16*>(q_mask), qcs, qbs, with_v ? 1 : 0, dm.L, dm.Hq, dm.Hkv,
        dm.flags, summary, entropy, with_v ? static_cast<__nv_bfloat16*>(o_mask) : nullptr);
    return cudaGetLastError();
  }
  if (std::is_same<T, __nv_bfloat16>::value && qcs % kVec == 0 && qbs % kVec == 0) {
    const size_t smem = (size_t)CONTENT * D * 2 * (with_v ? 2 : 1);
    auto kern = summary_pool_bulk_kernel<D>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(C, dm.Hkv, dm.B);
    count_launch();
    using B16 = __nv_bfloat16;
    kern<<<grid, 256, smem, st>>>(static_cast<const B16*>(q_mask), qcs, qbs, static_cast<const B16*>(k),
                                  with_v ? static_cast<const B16*>(v) : nullptr, dm.L, dm.Hq, dm.Hkv, dm.flags,
                                  summary, entropy, with_v ? static_cast<B16*>(o_mask) : nullptr);
    return cudaGetLastError();
  }
  const size_t smem = (size_t)(CONTENT * (D + 1) * (with_v ? 2 : 1) + 8 * D) * sizeof(float);
  auto kern = summary_pool_kernel<T, D>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(C, dm.Hkv, dm.B);
  count_launch();
  kern<<<grid, 256, smem, st>>>(static_cast<const T*>(q_mask), qcs, qbs, static_cast<const T*>(k),
                                with_v ? static_cast<const T*>(v) : nullptr, dm.L, dm.Hq, dm.Hkv,
                                dm.flags, summary, entropy,
                                with_v ? static_cast<T*>(o_mask) : nullptr);
  return cudaGetLastError();
}

}  // namespace rdl
