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

// ---------------------------------------------------------------------------
// Merge of the decode kernel's per-warp partial records (split-KV schedules).
// Row (b, h) of group g = b*Hkv + h/G collects the records of every piece of
// g: persistent schedule -> slots c + g for the CTAs c whose tile share meets
// g's tiles [T_g, T_g + n_g); split schedule -> slots g*S .. g*S + S-1.  Each
// record holds (O unnormalised, m in base 2, l, tiles); the merge is the same
// exact online-softmax combination as above, in base 2.
// ---------------------------------------------------------------------------
namespace skv {
namespace {

constexpr int kMaxRecords = 256;  // records per row handled by one warp (slots x warps)

__global__ void __launch_bounds__(kMergeWarps * 32) merge_records_kernel(const DecodeParams p, int G,
                                                                        int NW) {
  const int row = blockIdx.x * kMergeWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (row >= p.B * p.Hq) return;
  const int b = row / p.Hq, h = row % p.Hq, kvh = h / G, gh = h % G;
  const int g = b * p.Hkv + kvh;
  int s0 = 0, s1 = -1;  // slot range [s0, s1]
  long long T = 0, P = p.n_ctas;
  if (p.sched == SCHED_PERSISTENT) {
    T = p.ws_hdr[0];
    const int pb = p.ws_hdr[1 + b], pb1 = p.ws_hdr[2 + b];
    const int nt = (pb1 - pb) / p.Hkv;
    if (nt > 0 && T > 0) {
      const long long Tg = pb + (long long)kvh * nt;
      s0 = (int)(((Tg + 1) * P - 1) / T) + g;
      s1 = (int)(((Tg + nt) * P - 1) / T) + g;
    }
  } else {
    s0 = g * p.n_splits;
    s1 = s0 + p.n_splits - 1;
  }
  const int nrec = (s1 - s0 + 1) * NW;  // record r: slot s0 + r / NW, warp r % NW
  auto rec_ptr = [&](int r) {
    return p.ws_rec + (((size_t)(s0 + r / NW) * NW + (r % NW)) * G + gh) * kRecFloats;
  };
  auto rec_valid = [&](int r) {  // persistent: a CTA with an empty share wrote nothing
    if (p.sched != SCHED_PERSISTENT) return true;
    const long long c = s0 + r / NW - g;
    return (c * T) / P != ((c + 1) * T) / P;
  };
  // Records are combined in chunks of kMaxRecords: per chunk (1) m, l, tiles
  // spread over lanes and the chunk max, (2) weights 2^(m_r - M) and their
  // sum, (3) the weighted sum of the O vectors with four loads in flight;
  // chunks are folded into the running (M, W, acc) like any two partials.
  float M = -INFINITY, W = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  int tiles = 0;
  for (int base = 0; base < nrec; base += kMaxRecords) {
    const int cnt = min(kMaxRecords, nrec - base);
    float Mc = -INFINITY;
    float mr[kMaxRecords / 32], lr[kMaxRecords / 32];
#pragma unroll
    for (int u = 0; u < kMaxRecords / 32; ++u) {
      const int r = lane + 32 * u;
      mr[u] = -INFINITY;
      lr[u] = 0.f;
      if (r < cnt && rec_valid(base + r)) {
        const float4 ml = *reinterpret_cast<const float4*>(rec_ptr(base + r) + 128);  // m, l, tiles
        if (ml.y > 0.f) {
          mr[u] = ml.x;
          lr[u] = ml.y;
        }
        if ((base + r) % NW == 0) tiles += (int)ml.z;
      }
      Mc = fmaxf(Mc, mr[u]);
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) Mc = fmaxf(Mc, __shfl_xor_sync(0xffffffffu, Mc, m));
    if (Mc == -INFINITY) continue;
    float Wc = 0.f;
    float fr[kMaxRecords / 32];
#pragma unroll
    for (int u = 0; u < kMaxRecords / 32; ++u) {
      fr[u] = (lr[u] > 0.f) ? exp2f(mr[u] - Mc) : 0.f;
      Wc += fr[u] * lr[u];
    }
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) Wc += __shfl_xor_sync(0xffffffffu, Wc, m);
    float4 ac = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int u = 0; u < kMaxRecords / 32; ++u) {
      if (32 * u >= cnt) break;
      for (int r0 = 0; r0 < 32 && 32 * u + r0 < cnt; r0 += 4) {
        float4 o[4];
        float f[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int r = 32 * u + r0 + q;
          f[q] = __shfl_sync(0xffffffffu, fr[u], (r0 + q) & 31);
          o[q] = (r < cnt && f[q] > 0.f)
                     ? *reinterpret_cast<const float4*>(rec_ptr(base + r) + lane * 4)
                     : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          ac.x += f[q] * o[q].x;
          ac.y += f[q] * o[q].y;
          ac.z += f[q] * o[q].z;
          ac.w += f[q] * o[q].w;
        }
      }
    }
    const float mn = fmaxf(M, Mc);
    const float a = exp2f(M - mn), c = exp2f(Mc - mn);
    acc.x = acc.x * a + ac.x * c;
    acc.y = acc.y * a + ac.y * c;
    acc.z = acc.z * a + ac.z * c;
    acc.w = acc.w * a + ac.w * c;
    W = W * a + Wc * c;
    M = mn;
  }
#pragma unroll
  for (int m = 16; m >= 1; m >>= 1) tiles += __shfl_xor_sync(0xffffffffu, tiles, m);
  const float inv = (W > 0.f) ? 1.f / W : 0.f;
  *reinterpret_cast<float4*>(p.out + (size_t)row * kHeadDim + lane * 4) =
      make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
  if (lane == 0) {
    p.lse[row] = (W > 0.f) ? (M + log2f(W)) * 0.6931471805599453f : -INFINITY;
    if (p.blocks_consumed) p.blocks_consumed[row] = tiles;
  }
}

}  // namespace

int launch_merge_records(const DecodeParams& p, int G, void* stream) {
  const int N = p.B * p.Hq;
  if (N == 0) return 0;
  merge_records_kernel<<<(N + kMergeWarps - 1) / kMergeWarps, kMergeWarps * 32, 0,
                         static_cast<cudaStream_t>(stream)>>>(p, G, p.rec_nw);
  return (int)cudaGetLastError();
}

}  // namespace skv
