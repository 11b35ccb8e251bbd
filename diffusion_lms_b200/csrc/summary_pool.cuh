// Summary pooling: summary key s_c, pooling entropy H_c and the mask slot's own output
// (Prefilling-dLLM v2, Figure 3 caption: the mask's query pools the chunk's content keys
// with an intra-chunk softmax; the weighted sum is the summary key; the entropy of the
// pooling weights is the second routing signal).
//
// One CTA per (chunk c, KV head g, batch b): the chunk's 63 content keys (and values)
// are read from HBM once, staged in shared memory as fp32, and reused by every query
// head of the group.  The kernel streams K/V once, so it is HBM-bound.
#pragma once
#include "common.cuh"

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

template <typename T, int D>
cudaError_t launch_summary_pool(const void* q_mask, long long qcs, long long qbs, const void* k,
                                const void* v, const rdl_dims& dm, float* summary, float* entropy,
                                void* o_mask, cudaStream_t st) {
  const int C = dm.L / S;
  const bool with_v = v != nullptr && o_mask != nullptr;
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
