// tile.cuh -- the consumer-warp arithmetic of the decode kernels: one warp
// folds its slice of a 64-token KV tile into its online-softmax state
// (m, l, O) for the G query heads of a KV group ("ART" 2.1: tile-streaming
// attention exposes the partial output after every block).
//
// A warp owns RPW = 64 / NW consecutive rows of every tile.  Scores: a lane
// owns 8 dims of the K rows it visits and accumulates q.k for all G heads with
// packed fp32x2 FMAs; the partial sums are combined across the 16 lanes of a
// row by a select-free reduce-scatter (register r of lane L holds element
// r ^ X(L), so every level just adds the partner's upper half).  Exponentials
// are base 2 (q is pre-scaled by scale * log2 e).  P.V: a lane owns 4 output
// dims of every head; P is broadcast through shared memory as duplicated
// (p, p) pairs so that every FMA is a packed fp32x2 one.
//
// The tile pointers are generic: the kernels pass shared-memory stages, and
// the ART re-run passes pages of the pool in global memory.
#pragma once

#include "common.cuh"

namespace skv {
namespace {

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

template <int G, int NW>
struct Lanes {
  static constexpr int RPW = kBlock / NW;  // rows per warp per tile
  static constexpr int STEPS = RPW / 2;    // row steps per lane (two row parities)
  static constexpr int LG = ilog2(G);
  static constexpr int N = STEPS * G;      // partial dot products per lane
  static constexpr int LN = ilog2(N);
  static constexpr int S = LN < 4 ? LN : 4;  // reduce-scatter levels
  static constexpr int VPL = 1 << (LN - S);  // complete scores per lane
  static_assert(STEPS == 2 || STEPS == 4, "8 or 16 consumer warps");
  static_assert(G == 1 || G == 2 || G == 4 || G == 8, "group size");
};

// Select-free reduce-scatter over the 16 lanes of a row parity (register r of
// lane L holds element r ^ X(L)); levels beyond the scatter are all-reduces.
template <int N, int S>
__device__ __forceinline__ void reduce_scatter_xor(float (&v)[N]) {
  int n = N;
#pragma unroll
  for (int lvl = 0; lvl < 4; ++lvl) {
    const int m = 8 >> lvl;
    if (lvl < S) {
#pragma unroll
      for (int j = 0; j < N / 2; ++j)
        if (j < n / 2) v[j] += __shfl_xor_sync(0xffffffffu, v[j + n / 2], m);
      n >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
    }
  }
}

template <int STEPS>
__device__ __forceinline__ float rows_max(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
  if (STEPS == 4) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
  return x;
}
template <int STEPS>
__device__ __forceinline__ float rows_sum(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 16);
  x += __shfl_xor_sync(0xffffffffu, x, 8);
  if (STEPS == 4) x += __shfl_xor_sync(0xffffffffu, x, 4);
  return x;
}

// Per-warp consumer state.
template <int G, int NW>
struct Warp {
  using C = Lanes<G, NW>;
  f2 qf[G][4];        // register gr holds head gr ^ Xg, dims 8c .. 8c+7 (scaled)
  float m_st[C::VPL], l_st[C::VPL];
  f2 acc[G][2];       // O for dims 4*lane .. 4*lane+3 of every head (natural order)
  int hd[C::VPL];     // head of score slot j
  int lrow;           // local row (within the warp's slice) of the score slots
  int koff[C::STEPS]; // byte offsets of this lane's K chunk per row step
  int voff;           // byte offset of this lane's V chunk in row 0 of the slice
  int Xg;             // head relabelling of this lane's q registers
  bool owner;         // lane with row bits 0 (one of the writers of per-head scalars)

  __device__ __forceinline__ void setup(int warp, int lane) {
    const int c = lane & 15, par = lane >> 4;
    const int Xl = ((lane & 15) >> (4 - C::S)) << (C::LN - C::S);
    Xg = Xl & (G - 1);
    const int Xi = Xl >> C::LG;
    const int rb = warp * C::RPW;
#pragma unroll
    for (int i = 0; i < C::STEPS; ++i) koff[i] = (rb + par + 2 * (i ^ Xi)) * kRowBytes + c * 16;
    voff = rb * kRowBytes + lane * 8;
#pragma unroll
    for (int j = 0; j < C::VPL; ++j) hd[j] = (Xl + j) & (G - 1);
    lrow = par + 2 * (Xl >> C::LG);
    owner = (lane & (16 | (C::STEPS == 4 ? 12 : 8))) == 0;
  }

  __device__ __forceinline__ void reset() {
#pragma unroll
    for (int j = 0; j < C::VPL; ++j) {
      m_st[j] = -INFINITY;
      l_st[j] = 0.f;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) acc[g][0] = acc[g][1] = pack2(0.f, 0.f);
  }

  // Reset only the heads in `mask`.
  __device__ __forceinline__ void reset_heads(uint32_t mask) {
#pragma unroll
    for (int j = 0; j < C::VPL; ++j)
      if ((mask >> hd[j]) & 1u) {
        m_st[j] = -INFINITY;
        l_st[j] = 0.f;
      }
#pragma unroll
    for (int g = 0; g < G; ++g)
      if ((mask >> g) & 1u) acc[g][0] = acc[g][1] = pack2(0.f, 0.f);
  }

  // q of heads h0 .. h0+G-1 of sequence b (row stride: q_heads), pre-scaled.
  __device__ __forceinline__ void load_q(const uint16_t* q, size_t row0, float qscale, int lane) {
    const uint16_t* qrow = q + row0 * kHeadDim + (lane & 15) * 8;
#pragma unroll
    for (int gr = 0; gr < G; ++gr) {
      const uint4 w = *reinterpret_cast<const uint4*>(qrow + (size_t)(gr ^ Xg) * kHeadDim);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
        qf[gr][u] = pack2(__uint_as_float(ws[u] << 16) * qscale,
                          __uint_as_float(ws[u] & 0xFFFF0000u) * qscale);
    }
  }
};

// Fold this warp's rows of one tile.  nv: valid rows of the slice (MASKED:
// rows >= nv are ignored; their bytes are still read and must be readable).
// done_mask: heads that ignore the tile (state unchanged).
template <int G, int NW, bool MASKED>
__device__ __forceinline__ void fold_tile(Warp<G, NW>& W, const unsigned char* sK,
                                          const unsigned char* sV, int nv, uint32_t done_mask,
                                          float2* pbuf, float2* abuf) {
  using C = Lanes<G, NW>;
  // ---- scores
  float v[C::N];
  {
    f2 a2[C::STEPS][G];
#pragma unroll
    for (int i = 0; i < C::STEPS; ++i)
#pragma unroll
      for (int g = 0; g < G; ++g) a2[i][g] = pack2(0.f, 0.f);
#pragma unroll
    for (int i = 0; i < C::STEPS; ++i) {
      const uint4 w = *reinterpret_cast<const uint4*>(sK + W.koff[i]);
      const f2 k0 = bf2_to_f2(w.x), k1 = bf2_to_f2(w.y), k2 = bf2_to_f2(w.z), k3 = bf2_to_f2(w.w);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        ffma2(a2[i][g], W.qf[g][0], k0);
        ffma2(a2[i][g], W.qf[g][1], k1);
        ffma2(a2[i][g], W.qf[g][2], k2);
        ffma2(a2[i][g], W.qf[g][3], k3);
      }
    }
#pragma unroll
    for (int i = 0; i < C::STEPS; ++i)
#pragma unroll
      for (int g = 0; g < G; ++g) {
        float x, y;
        unpack2(a2[i][g], x, y);
        v[i * G + g] = x + y;
      }
  }
  reduce_scatter_xor<C::N, C::S>(v);

  // ---- online softmax (base 2)
#pragma unroll
  for (int j = 0; j < C::VPL; ++j) {
    const int g = W.hd[j];
    bool live = !((done_mask >> g) & 1u);
    if (MASKED) live = live && (W.lrow < nv);
    const float sv = live ? v[j] : -INFINITY;
    const float tmax = rows_max<C::STEPS>(sv);
    const float m_new = fmaxf(W.m_st[j], tmax);
    const float mu = (m_new == -INFINITY) ? 0.f : m_new;
    const float alpha = exp2f(W.m_st[j] - mu);
    const float pv = exp2f(sv - mu);
    W.l_st[j] = W.l_st[j] * alpha + rows_sum<C::STEPS>(pv);
    W.m_st[j] = m_new;
    pbuf[W.lrow * G + g] = make_float2(pv, pv);
    abuf[g] = make_float2(alpha, alpha);  // every lane of head g holds the same value
  }
  __syncwarp();

  // ---- O = alpha O + P V
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const float2 a = abuf[g];
    const f2 a2 = pack2(a.x, a.y);
    W.acc[g][0] = fmul2(W.acc[g][0], a2);
    W.acc[g][1] = fmul2(W.acc[g][1], a2);
  }
#pragma unroll
  for (int r = 0; r < C::RPW; ++r) {
    uint2 w = *reinterpret_cast<const uint2*>(sV + W.voff + r * kRowBytes);
    if (MASKED && r >= nv) w = make_uint2(0u, 0u);
    const f2 v0 = bf2_to_f2(w.x), v1 = bf2_to_f2(w.y);
    if constexpr (G == 1) {
      const float2 pp = pbuf[r];
      const f2 p2 = pack2(pp.x, pp.y);
      ffma2(W.acc[0][0], p2, v0);
      ffma2(W.acc[0][1], p2, v1);
    } else {
#pragma unroll
      for (int g2 = 0; g2 < G / 2; ++g2) {
        const float4 pp = *reinterpret_cast<const float4*>(pbuf + r * G + 2 * g2);
        const f2 pa = pack2(pp.x, pp.y), pb = pack2(pp.z, pp.w);
        ffma2(W.acc[2 * g2][0], pa, v0);
        ffma2(W.acc[2 * g2][1], pa, v1);
        ffma2(W.acc[2 * g2 + 1][0], pb, v0);
        ffma2(W.acc[2 * g2 + 1][1], pb, v1);
      }
    }
  }
  __syncwarp();
}

}  // namespace
}  // namespace skv
