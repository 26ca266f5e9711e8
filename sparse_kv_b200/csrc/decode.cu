// decode.cu -- streaming block-wise decode attention for sm_100a.
//
// One CTA per (KV group, split).  Warp 8 is the producer: one lane walks the
// traversal and issues bulk-async copies (TMA engine, cp.async.bulk) of the K
// and V rows of each tile (<= 64 consecutive tokens, <= 2 pages) into a
// STAGES-deep shared-memory ring guarded by full/empty mbarriers.  Warps 0..7
// consume: warp w owns rows 8w..8w+7 of every tile and keeps its own online
// softmax state (m, l, O) for the G query heads of the group
// ("ART" 2.1: tile-streaming attention exposes the partial state after every
// block).  Scores use packed fp32x2 FMAs over bf16 K rows, a 16-lane
// reduce-scatter, and base-2 exponentials; P.V uses packed FMAs too.
//
// With ART ("ART" 2.2-2.4) the eight warp states are combined after every
// tile into the probe x_t = (O/l)[0:8] of each head, the dual-threshold test
// with patience is evaluated (identically by every warp), and loads stop once
// all heads of the group have stopped.  Without ART, traversals are split
// across CTAs and the partials merged exactly (launch_merge).
#include "common.cuh"
#include "decode.cuh"

namespace skv {
namespace {

constexpr int kConsumerWarps = 8;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kStages = 5;
constexpr float kLn2 = 0.6931471805599453f;

// ---------------------------------------------------------------------------
// Traversal: yields tiles (t0, n) = n <= 64 consecutive tokens from t0, with
// the page(s) holding them.  Producer and consumers run identical copies.
// ---------------------------------------------------------------------------
struct Trav {
  int mode, L, nb;
  bool art;
  const int* bt;  // block_table row of this sequence
  int num_pages;
  // index-based modes
  int i, i_end;
  int ra, re;      // natural / range token interval
  int A, Rs, nt1;  // window: [0, A) then [Rs, L)
  const int* ord;
  int art_first;
  // segments
  const int* ss;
  const int* se;
  int seg_i, seg_end_i, seg_pos, seg_stop;

  __device__ void init(const DecodeParams& p, bool art_on, int b, int kvh, int L_, int split) {
    mode = p.mode;
    L = L_;
    nb = (L + kBlock - 1) / kBlock;
    art = art_on;
    bt = p.block_table + (size_t)b * p.max_blocks;
    num_pages = p.num_pages;
    ord = nullptr;
    art_first = 1;
    seg_pos = seg_stop = 0;
    const int grp = b * p.Hkv + kvh;
    int N = 0;
    if (mode == TRAV_NATURAL) {
      ra = 0;
      re = L;
      if (p.range_end > 0) {
        ra = max(p.range_begin, 0);
        re = min(p.range_end, L);
      }
      N = (re > ra) ? (re + kBlock - 1) / kBlock - ra / kBlock : 0;
    } else if (mode == TRAV_WINDOW) {
      A = min(p.sink, L);
      Rs = max(A, L - p.recent);
      nt1 = (A + kBlock - 1) / kBlock;
      N = nt1 + ((L > Rs) ? nb - Rs / kBlock : 0);
    } else if (mode == TRAV_ORDER) {
      ord = p.order + (size_t)grp * p.order_len;
      N = p.order_len;
    } else {  // segments
      ss = p.seg_start + (size_t)grp * p.n_seg;
      se = p.seg_end + (size_t)grp * p.n_seg;
      N = p.n_seg;
    }
    if (art) {  // one CTA walks the whole traversal
      if (mode == TRAV_ORDER) {
        i = 0;
        i_end = p.order_len;
      } else {
        i = nb - 1;  // recency-first countdown
        i_end = 0;
      }
      return;
    }
    const int S = p.n_splits;
    const int lo = (int)(((long long)split * N) / S), hi = (int)(((long long)(split + 1) * N) / S);
    if (mode == TRAV_SEGMENTS) {
      seg_i = lo;
      seg_end_i = hi;
    } else {
      i = lo;
      i_end = hi;
    }
  }

  __device__ bool next(int& t0, int& n, int& pg1, int& pg2, int& n1, uint32_t* status) {
    while (true) {
      int a, e;
      if (mode == TRAV_SEGMENTS) {
        if (seg_pos >= seg_stop) {
          if (seg_i >= seg_end_i) return false;
          int s = ss[seg_i], t = se[seg_i];
          ++seg_i;
          if (s > t) {
            dev_error(status, SKV_DEV_BAD_SEGMENT);
            continue;
          }
          seg_pos = max(s, 0);
          seg_stop = min(t, L);
          continue;
        }
        a = seg_pos;
        e = min(seg_pos + kBlock, seg_stop);
        seg_pos = e;
      } else if (art || mode == TRAV_ORDER) {
        int j;
        if (art && art_first) {
          art_first = 0;
          if (nb == 0) return false;
          j = 0;
        } else if (mode == TRAV_ORDER) {
          if (i >= i_end) return false;
          j = ord[i++];
          if (art && j == 0) continue;
          if (j < 0 || j >= nb) {
            dev_error(status, SKV_DEV_BAD_ORDER);
            continue;
          }
        } else {  // ART, recency-first
          if (i < 1) return false;
          j = i--;
        }
        a = j * kBlock;
        e = min(a + kBlock, L);
      } else {
        if (i >= i_end) return false;
        const int idx = i++;
        if (mode == TRAV_NATURAL) {
          const int j = ra / kBlock + idx;
          a = max(j * kBlock, ra);
          e = min(j * kBlock + kBlock, re);
        } else {  // window
          if (idx < nt1) {
            a = idx * kBlock;
            e = min(a + kBlock, A);
          } else {
            const int j = Rs / kBlock + (idx - nt1);
            a = max(j * kBlock, Rs);
            e = min(j * kBlock + kBlock, L);
          }
        }
      }
      n = e - a;
      if (n <= 0) continue;
      t0 = a;
      const int blk = a / kBlock, r0 = a % kBlock;
      n1 = min(kBlock - r0, n);
      pg1 = bt[blk];
      pg2 = (n > n1) ? bt[blk + 1] : 0;
      if (pg1 < 0 || pg1 >= num_pages || pg2 < 0 || pg2 >= num_pages) {
        dev_error(status, SKV_DEV_BAD_PAGE);
        continue;
      }
      return true;
    }
  }
};

template <int G>
struct Smem {
  static constexpr int kVpl = (4 * G >= 16) ? (4 * G / 16) : 1;  // scores per lane
  static constexpr size_t kStageBytes = 2 * kTileBytes;
  static constexpr size_t off_bar = kStages * kStageBytes;  // full[S], empty[S], probe[2], fin
  static constexpr size_t off_flags = off_bar + (2 * kStages + 3) * 8;  // int[8]
  static constexpr size_t off_p = (off_flags + 32 + 15) / 16 * 16;  // float2 [8 warps][8 rows][G]
  static constexpr size_t off_a = off_p + kConsumerWarps * 8 * G * 8;       // float2 [8][G]
  static constexpr size_t off_probe = off_a + kConsumerWarps * G * 8;       // float [2][8][G][10]
  static constexpr size_t off_fin = off_probe + 2 * kConsumerWarps * G * 10 * 4;  // float [8][G][128]
  static constexpr size_t off_finml = off_fin + kConsumerWarps * G * kHeadDim * 4;  // float [8][G][2]
  static constexpr size_t total = off_finml + kConsumerWarps * G * 2 * 4;
};

// Reduce-scatter of N partial sums across the 16 lanes sharing a row parity:
// afterwards lane holds the complete sums of elements e0 .. e0 + N/16 - 1
// (or, for N < 16, one element replicated over the remaining lanes).
template <int N>
__device__ __forceinline__ void reduce_scatter16(float (&v)[N], int lane) {
  int n = N;
#pragma unroll
  for (int m = 8; m >= 1; m >>= 1) {
    if (n > 1) {
      const bool up = (lane & m) != 0;
#pragma unroll
      for (int j = 0; j < N / 2; ++j) {
        if (j < n / 2) {
          const float send = up ? v[j] : v[j + n / 2];
          const float keep = up ? v[j + n / 2] : v[j];
          v[j] = keep + __shfl_xor_sync(0xffffffffu, send, m);
        }
      }
      n >>= 1;
    } else {
      v[0] += __shfl_xor_sync(0xffffffffu, v[0], m);
    }
  }
}

template <int N>
__device__ __forceinline__ int scatter_base(int lane) {
  int n = N, e = 0;
#pragma unroll
  for (int m = 8; m >= 1; m >>= 1) {
    if (n > 1) {
      if (lane & m) e += n / 2;
      n >>= 1;
    }
  }
  return e;
}

__device__ __forceinline__ float xor_max_rows(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 4));
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 8));
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 16));
  return x;
}
__device__ __forceinline__ float xor_sum_rows(float x) {
  x += __shfl_xor_sync(0xffffffffu, x, 4);
  x += __shfl_xor_sync(0xffffffffu, x, 8);
  x += __shfl_xor_sync(0xffffffffu, x, 16);
  return x;
}

template <int G, bool ART>
__global__ void __launch_bounds__(kThreads, 1) decode_kernel(const DecodeParams p) {
  using SM = Smem<G>;
  constexpr int VPL = SM::kVpl;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + SM::off_bar);
  uint64_t* empty = full + kStages;
  uint64_t* probe_bar = empty + kStages;  // [2], one arrival per consumer warp
  uint64_t* fin_bar = probe_bar + 2;      // one arrival per consumer warp
  volatile int* flags = reinterpret_cast<volatile int*>(smem + SM::off_flags);
  // flags[0]: ART stop (tiles consumed + 1; 0 = running)
  // flags[1]: abort (a bounded wait expired)
  // flags[2]: consumers finished (tiles consumed + 1; 0 = running)

  const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  int L = p.seq_lens[b];
  if (L < 0 || L > p.max_seq_len) {
    if (threadIdx.x == 0) dev_error(p.status, SKV_DEV_BAD_SEQLEN);
    L = 0;
  }

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kConsumerWarps);
    }
    mbar_init(&probe_bar[0], kConsumerWarps);
    mbar_init(&probe_bar[1], kConsumerWarps);
    mbar_init(fin_bar, kConsumerWarps);
    flags[0] = 0;
    flags[1] = 0;
    flags[2] = 0;
    fence_barrier_init();
  }
  __syncthreads();

  Trav tr;
  tr.init(p, ART, b, kvh, L, split);

  // ------------------------------------------------------------------ producer
  if (warp == kConsumerWarps) {
    if (lane == 0) {
      const uint64_t pol = policy_evict_first();
      const size_t head_stride = (size_t)kBlock * kHeadDim;  // elements per (page, head)
      int k = 0;
      int t0, n, pg1, pg2, n1;
      bool aborted = false;
      while (tr.next(t0, n, pg1, pg2, n1, p.status)) {
        if (flags[0] != 0) break;
        const int s = k % kStages;
        if (k >= kStages) {
          const uint32_t par = ((k / kStages) - 1) & 1;
          uint64_t t_start = 0;
          bool ok = true;
          while (!mbar_try_wait(&empty[s], par)) {
            if (flags[0] != 0 || flags[1] != 0) { ok = false; break; }
            const uint64_t now = globaltimer();
            if (t_start == 0) t_start = now;
            else if (now - t_start > kWaitLimitNs) {
              dev_error(p.status, SKV_DEV_TIMEOUT);
              flags[1] = 1;
              ok = false;
              break;
            }
          }
          if (!ok) { aborted = flags[1] != 0; break; }
        }
        unsigned char* sK = smem + s * SM::kStageBytes;
        unsigned char* sV = sK + kTileBytes;
        const uint32_t bytes = (uint32_t)n * kRowBytes * 2;
        mbar_arrive_expect_tx(&full[s], bytes);
        const int r0 = t0 % kBlock;
        const size_t src1 = ((size_t)pg1 * p.Hkv + kvh) * head_stride + (size_t)r0 * kHeadDim;
        bulk_load(sK, p.k_pool + src1, (uint32_t)n1 * kRowBytes, &full[s], pol);
        bulk_load(sV, p.v_pool + src1, (uint32_t)n1 * kRowBytes, &full[s], pol);
        if (n > n1) {
          const size_t src2 = ((size_t)pg2 * p.Hkv + kvh) * head_stride;
          bulk_load(sK + n1 * kRowBytes, p.k_pool + src2, (uint32_t)(n - n1) * kRowBytes, &full[s], pol);
          bulk_load(sV + n1 * kRowBytes, p.v_pool + src2, (uint32_t)(n - n1) * kRowBytes, &full[s], pol);
        }
        ++k;
      }
      // Copies the consumers never waited for (ART stop, abort) must land before
      // the CTA exits: learn how many tiles they consumed, then drain the rest.
      const uint64_t t_start = globaltimer();
      while (flags[2] == 0 && globaltimer() - t_start < kWaitLimitNs) {
      }
      int consumed = flags[2] - 1;
      if (consumed < 0 || aborted || flags[1] != 0) consumed = 0;
      for (int kk = (k - kStages > consumed ? k - kStages : consumed); kk < k; ++kk)
        mbar_wait_bounded(&full[kk % kStages], (kk / kStages) & 1, nullptr);
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  // Lane roles for Q.K: 16-byte chunk c (dims 8c..8c+7) of rows 8*warp + par + 2i.
  const int c = lane & 15, par = lane >> 4;
  const int h0 = kvh * G;
  f2 qf[G][4];
  {
    const uint16_t* qrow = p.q + ((size_t)b * p.Hq + h0) * kHeadDim + c * 8;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const uint4 w = *reinterpret_cast<const uint4*>(qrow + (size_t)g * kHeadDim);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        qf[g][u] = pack2(__uint_as_float(ws[u] << 16) * p.qscale,
                         __uint_as_float(ws[u] & 0xFFFF0000u) * p.qscale);
      }
    }
  }
  const int e0 = scatter_base<4 * G>(lane);
  // head of score slot k, local row of the slot
  int hd[VPL];
#pragma unroll
  for (int k = 0; k < VPL; ++k) hd[k] = (e0 + k) % G;
  const int lrow = par + 2 * (e0 / G);  // all VPL slots share the row

  float m_st[VPL], l_st[VPL];
#pragma unroll
  for (int k = 0; k < VPL; ++k) {
    m_st[k] = -INFINITY;
    l_st[k] = 0.f;
  }
  f2 acc[G][2];
#pragma unroll
  for (int g = 0; g < G; ++g) acc[g][0] = acc[g][1] = pack2(0.f, 0.f);

  float2* pbuf = reinterpret_cast<float2*>(smem + SM::off_p) + warp * 8 * G;
  float2* abuf = reinterpret_cast<float2*>(smem + SM::off_a) + warp * G;
  float* probe = reinterpret_cast<float*>(smem + SM::off_probe);

  // ART state (identical in every consumer warp)
  uint32_t done_mask = 0;  // bit g: head g stopped
  int cnt[G];
  int used[G];
  float xprev[(G + 3) / 4];
#pragma unroll
  for (int g = 0; g < G; ++g) { cnt[g] = 0; used[g] = 0; }
#pragma unroll
  for (int u = 0; u < (G + 3) / 4; ++u) xprev[u] = 0.f;

  int k = 0;
  int t0, n, pg1, pg2, n1;
  while (tr.next(t0, n, pg1, pg2, n1, nullptr)) {
    const int s = k % kStages;
    if (!mbar_wait_bounded(&full[s], (k / kStages) & 1, &flags[1])) {
      if (lane == 0) {
        dev_error(p.status, SKV_DEV_TIMEOUT);
        flags[1] = 1;
      }
      break;
    }
    const unsigned char* sK = smem + s * SM::kStageBytes;
    const unsigned char* sV = sK + kTileBytes;
    const int nrow_w = n - 8 * warp;  // valid rows of this warp's slice (may be <= 0)

    // ---- scores
    float sc[4 * G];
    {
      f2 a2[4][G];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int g = 0; g < G; ++g) a2[i][g] = pack2(0.f, 0.f);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int row = 8 * warp + par + 2 * i;
        const uint4 w = *reinterpret_cast<const uint4*>(sK + row * kRowBytes + c * 16);
        const f2 k0 = bf2_to_f2(w.x), k1 = bf2_to_f2(w.y), k2 = bf2_to_f2(w.z), k3 = bf2_to_f2(w.w);
#pragma unroll
        for (int g = 0; g < G; ++g) {
          ffma2(a2[i][g], qf[g][0], k0);
          ffma2(a2[i][g], qf[g][1], k1);
          ffma2(a2[i][g], qf[g][2], k2);
          ffma2(a2[i][g], qf[g][3], k3);
        }
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float x, y;
          unpack2(a2[i][g], x, y);
          sc[i * G + g] = x + y;
        }
    }
    reduce_scatter16<4 * G>(sc, lane);

    // ---- online softmax (base 2), per score slot
    const bool row_ok = lrow < nrow_w;
#pragma unroll
    for (int kk = 0; kk < VPL; ++kk) {
      const int g = hd[kk];
      const bool live = row_ok && !((done_mask >> g) & 1u);
      const float sv = live ? sc[kk] : -INFINITY;
      const float tmax = xor_max_rows(sv);
      const float m_new = fmaxf(m_st[kk], tmax);
      const float mu = (m_new == -INFINITY) ? 0.f : m_new;
      const float alpha = exp2f(m_st[kk] - mu);
      const float pv = exp2f(sv - mu);
      const float psum = xor_sum_rows(pv);
      l_st[kk] = l_st[kk] * alpha + psum;
      m_st[kk] = m_new;
      pbuf[lrow * G + g] = make_float2(pv, pv);
      if ((lane & 0x1C) == 0) abuf[g] = make_float2(alpha, alpha);
    }
    __syncwarp();

    // ---- O = alpha * O + P V   (lane owns dims 4*lane .. 4*lane+3)
#pragma unroll
    for (int g = 0; g < G; ++g) {
      const float2 a = abuf[g];
      const f2 a2 = pack2(a.x, a.y);
      acc[g][0] = fmul2(acc[g][0], a2);
      acc[g][1] = fmul2(acc[g][1], a2);
    }
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      const int row = 8 * warp + r;
      uint2 w = *reinterpret_cast<const uint2*>(sV + row * kRowBytes + lane * 8);
      if (r >= nrow_w) w = make_uint2(0u, 0u);
      const f2 v0 = bf2_to_f2(w.x), v1 = bf2_to_f2(w.y);
#pragma unroll
      for (int g = 0; g < G; ++g) {
        const float2 pp = pbuf[r * G + g];
        const f2 p2 = pack2(pp.x, pp.y);
        ffma2(acc[g][0], p2, v0);
        ffma2(acc[g][1], p2, v1);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);

    if constexpr (ART) {
      // ---- probe exchange: (m, l, O[0:8]) of every warp and head
      float* pb = probe + (k & 1) * (kConsumerWarps * G * 10) + warp * G * 10;
      if (lane < 4) {
#pragma unroll
        for (int kk = 0; kk < VPL; ++kk) {
          pb[hd[kk] * 10 + 0] = m_st[kk];
          pb[hd[kk] * 10 + 1] = l_st[kk];
        }
      }
      if (lane < 2) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float x0, x1, x2, x3;
          unpack2(acc[g][0], x0, x1);
          unpack2(acc[g][1], x2, x3);
          pb[g * 10 + 2 + lane * 4 + 0] = x0;
          pb[g * 10 + 2 + lane * 4 + 1] = x1;
          pb[g * 10 + 2 + lane * 4 + 2] = x2;
          pb[g * 10 + 2 + lane * 4 + 3] = x3;
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&probe_bar[k & 1]);
      if (!mbar_wait_bounded(&probe_bar[k & 1], (k >> 1) & 1, &flags[1])) {
        if (lane == 0) {
          dev_error(p.status, SKV_DEV_TIMEOUT);
          flags[1] = 1;
        }
        break;
      }
      const float* pall = probe + (k & 1) * (kConsumerWarps * G * 10);
      uint32_t pass_mask = 0;
#pragma unroll
      for (int u = 0; u < (G + 3) / 4; ++u) {
        const int g = u * 4 + (lane >> 3), e = lane & 7;
        float x = 0.f;
        if (g < G) {
          float M = -INFINITY;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, pall[(w * G + g) * 10]);
          float Ls = 0.f, X = 0.f;
          if (M != -INFINITY) {
#pragma unroll
            for (int w = 0; w < kConsumerWarps; ++w) {
              const float f = exp2f(pall[(w * G + g) * 10] - M);
              Ls += pall[(w * G + g) * 10 + 1] * f;
              X += pall[(w * G + g) * 10 + 2 + e] * f;
            }
          }
          x = (Ls > 0.f) ? X / Ls : 0.f;
        }
        // norms and the direction change of unit vectors, over the 8 lanes of a head
        float nx = x * x, np = xprev[u] * xprev[u];
#pragma unroll
        for (int m = 1; m < 8; m <<= 1) {
          nx += __shfl_xor_sync(0xffffffffu, nx, m);
          np += __shfl_xor_sync(0xffffffffu, np, m);
        }
        const float a = sqrtf(nx), bp = sqrtf(np);
        const float du = ((a > 0.f) ? x / a : 0.f) - ((bp > 0.f) ? xprev[u] / bp : 0.f);
        float dd = du * du;
#pragma unroll
        for (int m = 1; m < 8; m <<= 1) dd += __shfl_xor_sync(0xffffffffu, dd, m);
        float d_s, d_c;
        if (bp == 0.f) d_s = (a == 0.f) ? 0.f : INFINITY;
        else d_s = fabsf(a - bp) / bp;
        if (a == 0.f || bp == 0.f) d_c = (a == 0.f && bp == 0.f) ? 0.f : 1.f;
        else d_c = 0.5f * dd;  // 1 - cos(x, x') = |x/|x| - x'/|x'||^2 / 2
        const bool pass = (k >= 1) && (d_s < p.tau) && (d_c < p.phi);
        const uint32_t bal = __ballot_sync(0xffffffffu, pass && e == 0 && g < G);
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4)
          if ((bal >> (q4 * 8)) & 1u) pass_mask |= 1u << (u * 4 + q4);
        xprev[u] = x;
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        if ((done_mask >> g) & 1u) continue;
        cnt[g] = ((pass_mask >> g) & 1u) ? cnt[g] + 1 : 0;
        if (cnt[g] >= p.patience) {
          done_mask |= 1u << g;
          used[g] = k + 1;
        }
      }
      if (done_mask == (1u << G) - 1u) {
        if (warp == 0 && lane == 0) flags[0] = k + 2;  // tiles consumed + 1
        ++k;
        break;
      }
    }
    ++k;
  }

  // ------------------------------------------------------------------ epilogue
  float* fin = reinterpret_cast<float*>(smem + SM::off_fin);
  float* finml = reinterpret_cast<float*>(smem + SM::off_finml);
  if (lane < 4) {
#pragma unroll
    for (int kk = 0; kk < VPL; ++kk) {
      finml[(warp * G + hd[kk]) * 2 + 0] = m_st[kk];
      finml[(warp * G + hd[kk]) * 2 + 1] = l_st[kk];
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    float x0, x1, x2, x3;
    unpack2(acc[g][0], x0, x1);
    unpack2(acc[g][1], x2, x3);
    *reinterpret_cast<float4*>(fin + (warp * G + g) * kHeadDim + lane * 4) = make_float4(x0, x1, x2, x3);
  }
  __syncwarp();
  if (lane == 0) mbar_arrive(fin_bar);
  if (!mbar_wait_bounded(fin_bar, 0, nullptr)) {
    if (lane == 0) dev_error(p.status, SKV_DEV_TIMEOUT);
  }
  if (threadIdx.x == 0) flags[2] = (flags[1] != 0) ? 1 : k + 1;
  const int nthr = kConsumerWarps * 32;
  for (int o = threadIdx.x; o < G * kHeadDim; o += nthr) {
    const int g = o / kHeadDim, dim = o % kHeadDim;
    float M = -INFINITY;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, finml[(w * G + g) * 2]);
    float Ls = 0.f, X = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) {
        const float f = exp2f(finml[(w * G + g) * 2] - M);
        Ls += finml[(w * G + g) * 2 + 1] * f;
        X += fin[(w * G + g) * kHeadDim + dim] * f;
      }
    }
    const float outv = (Ls > 0.f) ? X / Ls : 0.f;
    const float lsev = (Ls > 0.f) ? (M + log2f(Ls)) * kLn2 : -INFINITY;
    const size_t row = (size_t)b * p.Hq + h0 + g;
    if (p.n_splits > 1) {
      const size_t NR = (size_t)p.B * p.Hq;
      p.ws_o[((size_t)split * NR + row) * kHeadDim + dim] = outv;
      if (dim == 0) p.ws_lse[(size_t)split * NR + row] = lsev;
    } else {
      p.out[row * kHeadDim + dim] = outv;
      if (dim == 0) p.lse[row] = lsev;
    }
    if (dim == 0 && p.blocks_consumed) {
      if (ART) p.blocks_consumed[row] = ((done_mask >> g) & 1u) ? used[g] : k;
      else atomicAdd(&p.blocks_consumed[row], k);
    }
  }
}

template <int G, bool ART>
int launch_t(const DecodeParams& p, cudaStream_t st) {
  constexpr size_t smem = Smem<G>::total;
  auto kern = decode_kernel<G, ART>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return (int)e;
  dim3 grid(p.n_splits, p.Hkv, p.B);
  kern<<<grid, kThreads, smem, st>>>(p);
  return (int)cudaGetLastError();
}

}  // namespace

int launch_decode(const DecodeParams& p, int G, bool art, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (G) {
    case 1: return art ? launch_t<1, true>(p, st) : launch_t<1, false>(p, st);
    case 2: return art ? launch_t<2, true>(p, st) : launch_t<2, false>(p, st);
    case 4: return art ? launch_t<4, true>(p, st) : launch_t<4, false>(p, st);
    case 8: return art ? launch_t<8, true>(p, st) : launch_t<8, false>(p, st);
    default: return (int)cudaErrorInvalidValue;
  }
}

int num_sms() {
  static int cached = 0;
  if (cached == 0) {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && n > 0)
      cached = n;
    else
      return 148;
  }
  return cached;
}

}  // namespace skv
