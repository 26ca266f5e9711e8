// route.cu -- per-layer hard routing between full and sparse attention
// ("Flux Attention" section 2: a Layer Router pools the first and last tokens
// of the input query tensor and decides, per layer, full attention or sparse
// attention; at inference the soft decision is made hard, once per prefill).
// The router's weights are inputs: the pages train them, nothing here does.
//
// For layer l and sequence b, with F = q_heads * head_dim features per token:
//   f = [ mean of the first n_prefix query rows , mean of the last n_suffix ]
//   z = w_l . f + bias_l,      route = z > 0   (1: full attention)
//
// One CTA per (sequence, layer) streams its n_prefix + n_suffix rows with
// 16-byte loads: a thread owns one 8-feature chunk of every row (consecutive
// threads on consecutive bytes) and keeps eight rows in flight, the prefix
// and suffix rows walked as one list; it holds both running sums in registers
// and the block reduces the dot product.
// HBM-bound: (n_prefix + n_suffix) * F * 2 bytes of queries and 2 * F * 4
// bytes of weights per CTA.
#include <cuda_runtime.h>

#include "../../include/sparsekv.h"
#include "common.cuh"

namespace skv {
namespace {

constexpr int kRouteThreads = 512;  // 8-feature chunks per pass (F = 4096: one pass)
constexpr int kRouteRows = 8;       // rows in flight per thread (two CTAs per SM)

__device__ __forceinline__ void add_bf16x8(float (&s)[8], uint4 v) {
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    s[2 * i] += __uint_as_float(u[i] << 16);
    s[2 * i + 1] += __uint_as_float(u[i] & 0xFFFF0000u);
  }
}

__global__ void __launch_bounds__(kRouteThreads, 2) route_kernel(const uint16_t* __restrict__ q,
                                                             const float* __restrict__ w,
                                                             const float* __restrict__ bias, int B, int T,
                                                             int F, int n_prefix, int n_suffix,
                                                             float* __restrict__ logits,
                                                             uint8_t* __restrict__ route) {
  const int b = blockIdx.x, l = blockIdx.y;
  const uint16_t* qb = q + ((size_t)l * B + b) * (size_t)T * F;
  const float* wl = w + (size_t)l * 2 * F;
  const float inv_p = 1.f / (float)n_prefix, inv_s = 1.f / (float)n_suffix;
  float part = 0.f;
  const int n_rows = n_prefix + n_suffix;  // row r < n_prefix: prefix row r; else suffix row
  for (int c = threadIdx.x; c < F / 8; c += kRouteThreads) {
    float sp[8], ss[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) sp[j] = ss[j] = 0.f;
    const uint16_t* col = qb + (size_t)c * 8;
    for (int r0 = 0; r0 < n_rows; r0 += kRouteRows) {
      uint4 v[kRouteRows];
#pragma unroll
      for (int u = 0; u < kRouteRows; ++u) {
        const int r = r0 + u;
        const int t = r < n_prefix ? r : T - n_suffix + (r - n_prefix);
        v[u] = (r < n_rows) ? __ldg(reinterpret_cast<const uint4*>(col + (size_t)t * F))
                            : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kRouteRows; ++u) {
        if (r0 + u < n_prefix) add_bf16x8(sp, v[u]);
        else add_bf16x8(ss, v[u]);
      }
    }
    const float4 wp0 = __ldg(reinterpret_cast<const float4*>(wl + c * 8));
    const float4 wp1 = __ldg(reinterpret_cast<const float4*>(wl + c * 8 + 4));
    const float4 ws0 = __ldg(reinterpret_cast<const float4*>(wl + F + c * 8));
    const float4 ws1 = __ldg(reinterpret_cast<const float4*>(wl + F + c * 8 + 4));
    const float wp[8] = {wp0.x, wp0.y, wp0.z, wp0.w, wp1.x, wp1.y, wp1.z, wp1.w};
    const float ws[8] = {ws0.x, ws0.y, ws0.z, ws0.w, ws1.x, ws1.y, ws1.z, ws1.w};
#pragma unroll
    for (int j = 0; j < 8; ++j) part += sp[j] * inv_p * wp[j] + ss[j] * inv_s * ws[j];
  }
  // block reduction of the dot product
  __shared__ float red[kRouteThreads / 32];
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = part;
  __syncthreads();
  if (threadIdx.x == 0) {
    float z = 0.f;
#pragma unroll
    for (int i = 0; i < kRouteThreads / 32; ++i) z += red[i];
    if (bias) z += bias[l];
    if (logits) logits[(size_t)l * B + b] = z;
    route[(size_t)l * B + b] = z > 0.f ? 1 : 0;
  }
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace skv

extern "C" {

SKV_API skv_status attn_route_layers(const void* q, const float* w, const float* bias, int n_layers,
                                     int batch, int tokens, int q_heads, int head_dim, int n_prefix,
                                     int n_suffix, float* logits, uint8_t* route, skv_stream_t stream) {
  using namespace skv;
  if (!q || !w || !route) return SKV_EINVAL;
  if (n_layers < 1 || batch < 1 || tokens < 1 || q_heads < 1 || head_dim < 1) return SKV_EINVAL;
  if (n_prefix < 1 || n_prefix > tokens || n_suffix < 1 || n_suffix > tokens) return SKV_EINVAL;
  const long long F = (long long)q_heads * head_dim;
  if (F % 8 != 0 || F > (1 << 24)) return SKV_EUNSUPPORTED;
  if (n_layers > 65535 || batch > (1 << 30)) return SKV_EUNSUPPORTED;
  if (!aligned16(q) || !aligned16(w)) return SKV_EINVAL;
  route_kernel<<<dim3(batch, n_layers), kRouteThreads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint16_t*>(q), w, bias, batch, tokens, (int)F, n_prefix, n_suffix, logits, route);
  return cudaGetLastError() == cudaSuccess ? SKV_OK : SKV_ECUDA;
}

}  // extern "C"
