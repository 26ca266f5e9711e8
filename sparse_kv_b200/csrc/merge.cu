// merge.cu -- exact log-sum-exp merge of attention partials
// ("Pulsar Attention" Phase 2: per-shard local attention combined by the
// online-softmax merge into the exact global result).
//
// One warp per output row; lane j owns dims 4j.. (float4), looping for
// head_dim > 128.  HBM-bound: reads S*(d+1) floats and writes d+1 per row.
#include "common.cuh"
#include "decode.cuh"

namespace skv {
namespace {

constexpr int kMergeWarps = 8;

__global__ void __launch_bounds__(kMergeWarps * 32) merge_kernel(const float* __restrict__ o,
                                                               const float* __restrict__ l, int S,
                                                               int N, int d, float* __restrict__ out,
                                                               float* __restrict__ lse) {
  const int row = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= N) return;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, l[(size_t)s * N + row]);
  if (M == -INFINITY) {
    for (int j = lane * 4; j < d; j += 128)
      *reinterpret_cast<float4*>(out + (size_t)row * d + j) = make_float4(0.f, 0.f, 0.f, 0.f);
    if (lane == 0) lse[row] = -INFINITY;
    return;
  }
  float4 acc[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
  float W = 0.f;
  for (int s = 0; s < S; ++s) {
    const float w = expf(l[(size_t)s * N + row] - M);  // 0 for an empty partial
    W += w;
    if (w == 0.f) continue;
    const float* src = o + ((size_t)s * N + row) * d;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j = lane * 4 + u * 128;
      if (j < d) {
        const float4 v = *reinterpret_cast<const float4*>(src + j);
        acc[u].x += w * v.x;
        acc[u].y += w * v.y;
        acc[u].z += w * v.z;
        acc[u].w += w * v.w;
      }
    }
  }
  const float inv = 1.f / W;
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int j = lane * 4 + u * 128;
    if (j < d)
      *reinterpret_cast<float4*>(out + (size_t)row * d + j) =
          make_float4(acc[u].x * inv, acc[u].y * inv, acc[u].z * inv, acc[u].w * inv);
  }
  if (lane == 0) lse[row] = M + logf(W);
}

}  // namespace

int launch_merge(const float* o_parts, const float* lse_parts, int S, int N, int d, float* out,
                 float* lse, void* stream) {
  if (N == 0) return 0;
  const int blocks = (N + kMergeWarps - 1) / kMergeWarps;
  merge_kernel<<<blocks, kMergeWarps * 32, 0, static_cast<cudaStream_t>(stream)>>>(
      o_parts, lse_parts, S, N, d, out, lse);
  return (int)cudaGetLastError();
}

}  // namespace skv
