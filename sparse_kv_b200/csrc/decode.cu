// decode.cu -- streaming block-wise decode attention for sm_100a.
//
// Structure of a CTA: the last warp is the producer.  One of its lanes walks
// the traversal and issues bulk-async copies (TMA engine, cp.async.bulk, no
// multicast) of the K and V rows of each tile (<= 64 consecutive tokens from
// <= 2 pages) into a STAGES-deep shared-memory ring guarded by full/empty
// mbarriers, publishing each entry's row count and KV group in shared memory.
// NW consumer warps split every tile's 64 rows (64/NW each) and keep their own
// online-softmax state (m, l, O) for the G query heads of the group ("ART"
// 2.1: tile-streaming attention exposes the partial output after every block).
//
// Schedules.  Plain traversals run persistently: one CTA per SM takes an even
// share of the concatenated tile lists of all KV groups (a share may span
// group boundaries; consumers then write a partial record per warp and start
// the next group without any CTA-wide synchronisation).  Segment lists split
// each group across a fixed number of CTAs.  Both end with an exact merge of
// the per-warp records (launch_merge_records).  With ART, one CTA walks each
// group and writes the final output itself.
//
// Scores: a lane owns 8 dims of the K rows it visits and accumulates q.k for
// all G heads with packed fp32x2 FMAs; the partial sums are combined across
// the 16 lanes of a row by a select-free reduce-scatter (register r of lane L
// holds element r ^ X(L), so every level just adds the partner's upper half).
// Exponentials are base 2 (q is pre-scaled by scale * log2 e).  P.V: a lane
// owns 4 output dims of every head; P is broadcast through shared memory as
// duplicated (p, p) pairs so that every FMA is a packed fp32x2 one.
//
// ART ("ART" 2.2-2.4): after each tile every warp publishes (m, l, O[0:8]) per
// head; judge warp g (g < G) merges them into the probe x_t of head g, runs the
// dual-threshold test with patience and publishes the decision.  Decisions
// are applied two tiles later from a snapshot of the state after the decided
// tile, so the result is exactly the attention over the blocks up to the stop,
// and the judging overlaps the next tiles.  Loads stop once every head of the
// group has stopped.
#include "common.cuh"
#include "decode.cuh"

// Plain traversals: SKV_CONSUMER_WARPS consumer warps per CTA and
// SKV_CTAS_PER_SM resident CTAs per SM (both CTAs' warps hide each other's
// latency; fewer warps per tile means fewer per-warp fixed costs).  ART and
// 8-head groups use 8 warps and one CTA per SM (their state needs registers).
#ifndef SKV_CONSUMER_WARPS
#define SKV_CONSUMER_WARPS 8
#endif
#ifndef SKV_CTAS_PER_SM
#define SKV_CTAS_PER_SM 2
#endif
#ifndef SKV_CONSUMER_WARPS_ART
#define SKV_CONSUMER_WARPS_ART 8
#endif

namespace skv {
namespace {

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

  // Whole traversal of group (b, kvh); non-ART traversals are then narrowed
  // with set_range (index-based modes: tile indices; segments: segment indices).
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
    const int S = p.n_splits > 0 ? p.n_splits : 1;
    set_range((int)(((long long)split * N) / S), (int)(((long long)(split + 1) * N) / S));
  }

  __device__ void set_range(int lo, int hi) {
    if (mode == TRAV_SEGMENTS) {
      seg_i = lo;
      seg_end_i = hi;
      seg_pos = seg_stop = 0;
    } else {
      i = lo;
      i_end = hi;
    }
  }

  // Segment lists: the next piece = up to 64 consecutive tokens inside one
  // page (page, first row, rows).  Used to pack several segments into one tile.
  __device__ bool next_piece(int& page, int& r0, int& cnt, uint32_t* status) {
    while (true) {
      if (seg_pos >= seg_stop) {
        if (seg_i >= seg_end_i) return false;
        const int s = ss[seg_i], t = se[seg_i];
        ++seg_i;
        if (s > t) {
          dev_error(status, SKV_DEV_BAD_SEGMENT);
          continue;
        }
        seg_pos = max(s, 0);
        seg_stop = min(t, L);
        continue;
      }
      const int blk = seg_pos / kBlock;
      r0 = seg_pos % kBlock;
      cnt = min(kBlock - r0, seg_stop - seg_pos);
      seg_pos += cnt;
      page = bt[blk];
      if (page < 0 || page >= num_pages) {
        dev_error(status, SKV_DEV_BAD_PAGE);
        continue;
      }
      return true;
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

constexpr int ilog2(int x) { return x <= 1 ? 0 : 1 + ilog2(x / 2); }

template <int G, int NW, bool ART, int MINB>
struct Cfg {
  static constexpr int RPW = kBlock / NW;  // rows per warp per tile
  static constexpr int STEPS = RPW / 2;    // row steps per lane (two row parities)
  static constexpr int LG = ilog2(G);
  static constexpr int N = STEPS * G;      // partial dot products per lane
  static constexpr int LN = ilog2(N);
  static constexpr int S = LN < 4 ? LN : 4;  // reduce-scatter levels
  static constexpr int VPL = 1 << (LN - S);  // complete scores per lane
  static constexpr int STAGES = ART ? 5 : (MINB == 2 ? 3 : 6);
  static constexpr int THREADS = (NW + 1) * 32;
  static constexpr int PROBE = 12;  // floats per (warp, head) probe: m, l, pad, pad, O[0:8]
  static constexpr size_t STAGE_BYTES = 2 * (size_t)kTileBytes;
  static constexpr int NBAR = 2 * STAGES + 7;  // full, empty, probe[3], dec[3], fin
  static constexpr size_t OFF_BAR = STAGES * STAGE_BYTES;
  static constexpr size_t OFF_META = (OFF_BAR + NBAR * 8 + 15) / 16 * 16;   // int4 [STAGES]
  static constexpr size_t OFF_FLAGS = (OFF_META + STAGES * 16 + 15) / 16 * 16;
  static constexpr size_t OFF_DEC = OFF_FLAGS + 16;                       // int [3][G]
  static constexpr size_t OFF_P = (OFF_DEC + 3 * G * 4 + 15) / 16 * 16;  // float2 [NW][RPW][G]
  static constexpr size_t OFF_A = OFF_P + (size_t)NW * RPW * G * 8;        // float2 [NW][G]
  static constexpr size_t OFF_PROBE = OFF_A + (size_t)NW * G * 8;          // float [3][NW][G][12]
  static constexpr size_t N_PROBE = ART ? 3 * (size_t)NW * G * PROBE * 4 : 0;
  static constexpr size_t OFF_FIN = OFF_PROBE + N_PROBE;                   // float [NW][G][128]
  static constexpr size_t N_FIN = ART ? (size_t)NW * G * kHeadDim * 4 : 0;
  static constexpr size_t OFF_FINML = OFF_FIN + N_FIN;                     // float2 [NW][G]
  static constexpr size_t OFF_PRE = OFF_FINML + (ART ? (size_t)NW * G * 8 : 0);  // int [B+1], int [B]
  static constexpr size_t N_PRE = ART ? 0 : (2 * (size_t)kMaxPersistentBatch + 1) * 4;
  static constexpr size_t TOTAL = OFF_PRE + N_PRE;
  static_assert(TOTAL <= (MINB == 2 ? 113 : 227) * 1024, "shared memory budget");
  // every region read or written with 16-byte vectors starts 16-byte aligned
  static_assert(OFF_BAR % 16 == 0 && OFF_META % 16 == 0 && OFF_FLAGS % 16 == 0, "alignment");
  static_assert(OFF_P % 16 == 0 && OFF_A % 16 == 0 && OFF_PROBE % 16 == 0, "alignment");
  static_assert(OFF_FIN % 16 == 0 && OFF_FINML % 16 == 0 && OFF_PRE % 16 == 0, "alignment");
  static_assert((RPW * G * 8) % 16 == 0 || G == 1, "pbuf rows");
  static_assert((PROBE * 4) % 16 == 0 && (kRecFloats * 4) % 16 == 0, "record strides");
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
template <int G, int NW, bool ART, int MINB>
struct Warp {
  using C = Cfg<G, NW, ART, MINB>;
  f2 qf[G][4];        // register gr holds head gr ^ Xg, dims 8c .. 8c+7 (scaled)
  float m_st[C::VPL], l_st[C::VPL];
  f2 acc[G][2];       // O for dims 4*lane .. 4*lane+3 of every head (natural order)
  int hd[C::VPL];     // head of score slot j
  int lrow;           // local row (within the warp's slice) of the score slots
  int koff[C::STEPS]; // byte offsets of this lane's K chunk per row step
  int voff;           // byte offset of this lane's V chunk in row 0 of the slice
  bool owner;         // lane with row bits 0 (one of the writers of per-head scalars)
};

template <int G, int NW, bool ART, int MINB, bool MASKED>
__device__ __forceinline__ void fold_tile(Warp<G, NW, ART, MINB>& W, const unsigned char* sK,
                                          const unsigned char* sV, int nv, uint32_t done_mask,
                                          float2* pbuf, float2* abuf) {
  using C = Cfg<G, NW, ART, MINB>;
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


template <int G, bool ART, int NW, int MINB>
__global__ void __launch_bounds__(Cfg<G, NW, ART, MINB>::THREADS, MINB) decode_kernel(const DecodeParams p) {
  using C = Cfg<G, NW, ART, MINB>;
  constexpr int ST = C::STAGES;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + ST;
  uint64_t* probe_bar = empty + ST;   // [3], NW arrivals
  uint64_t* dec_bar = probe_bar + 3;  // [3], G arrivals
  uint64_t* fin_bar = dec_bar + 3;    // NW arrivals
  int4* meta = reinterpret_cast<int4*>(smem + C::OFF_META);  // {rows, group, slot, 0}
  volatile int* flags = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  // flags[0]: ART stop (entries consumed + 1; 0 = running)
  // flags[1]: abort (a bounded wait expired)
  // flags[2]: consumers finished (entries consumed + 1; 0 = running)
  volatile int* dec = reinterpret_cast<volatile int*>(smem + C::OFF_DEC);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NW);
    }
    for (int i = 0; i < 3; ++i) {
      mbar_init(&probe_bar[i], NW);
      mbar_init(&dec_bar[i], G);
    }
    mbar_init(fin_bar, NW);
    flags[0] = flags[1] = flags[2] = 0;
    fence_barrier_init();
  }
  __syncthreads();

  // ------------------------------------------------------------------ producer
  if (warp == NW) {
    int* pre = reinterpret_cast<int*>(smem + C::OFF_PRE);  // [B+1] tiles before batch b
    int* Lsm = pre + kMaxPersistentBatch + 1;              // [B] validated lengths
    if (!ART && p.sched == SCHED_PERSISTENT) {
      int run = 0;
      for (int base = 0; base < p.B; base += 32) {
        const int b = base + lane;
        int L = 0, t = 0;
        if (b < p.B) {
          L = p.seq_lens[b];
          if (L < 0 || L > p.max_seq_len) {
            if (blockIdx.x == 0) dev_error(p.status, SKV_DEV_BAD_SEQLEN);
            L = 0;
          }
          Lsm[b] = L;
          t = group_tiles(p, L) * p.Hkv;
        }
        int x = t;
#pragma unroll
        for (int m = 1; m < 32; m <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, x, m);
          if (lane >= m) x += y;
        }
        if (b < p.B) pre[b] = run + x - t;
        run += __shfl_sync(0xffffffffu, x, 31);
      }
      if (lane == 0) pre[p.B] = run;
      __syncwarp();
      if (blockIdx.x == 0) {
        if (lane == 0) p.ws_hdr[0] = run;
        for (int b = lane; b <= p.B; b += 32) p.ws_hdr[1 + b] = pre[b];
      }
    }
    if (lane != 0) return;

    const uint64_t pol = policy_evict_first();
    const size_t head_stride = (size_t)kBlock * kHeadDim;
    int e = 0, ps = 0, round = 0;  // entries issued, stage, ring round
    bool aborted = false;
    // Issue one ring entry: `n` rows of group `g` (n = 0: a group marker with
    // no rows, n = -1: end of traversal).  Returns false to stop issuing.
    auto emit = [&](int n, int g, int slot, int kvh, int t0, int pg1, int pg2, int n1) -> bool {
      if (round >= 1) {
        const uint32_t par = (round - 1) & 1;
        uint64_t t_start = 0;
        while (!mbar_try_wait(&empty[ps], par)) {
          if (flags[0] != 0 || flags[1] != 0) return false;
          const uint64_t now = globaltimer();
          if (t_start == 0) t_start = now;
          else if (now - t_start > kWaitLimitNs) {
            dev_error(p.status, SKV_DEV_TIMEOUT);
            flags[1] = 1;
            aborted = true;
            return false;
          }
        }
      }
      meta[ps] = make_int4(n, g, slot, 0);
      if (n > 0) {
        unsigned char* sK = smem + ps * C::STAGE_BYTES;
        unsigned char* sV = sK + kTileBytes;
        mbar_arrive_expect_tx(&full[ps], (uint32_t)n * kRowBytes * 2);
        const size_t src1 =
            ((size_t)pg1 * p.Hkv + kvh) * head_stride + (size_t)(t0 % kBlock) * kHeadDim;
        bulk_load(sK, p.k_pool + src1, (uint32_t)n1 * kRowBytes, &full[ps], pol);
        bulk_load(sV, p.v_pool + src1, (uint32_t)n1 * kRowBytes, &full[ps], pol);
        if (n > n1) {
          const size_t src2 = ((size_t)pg2 * p.Hkv + kvh) * head_stride;
          bulk_load(sK + n1 * kRowBytes, p.k_pool + src2, (uint32_t)(n - n1) * kRowBytes, &full[ps], pol);
          bulk_load(sV + n1 * kRowBytes, p.v_pool + src2, (uint32_t)(n - n1) * kRowBytes, &full[ps], pol);
        }
      } else {
        mbar_arrive(&full[ps]);
      }
      ++e;
      if (++ps == ST) {
        ps = 0;
        ++round;
      }
      return true;
    };
    // Segment lists: rows of several segments are packed into full 64-row
    // tiles (attention over a key set does not depend on the keys' order);
    // one bulk copy per piece (<= 64 consecutive tokens of one page).
    constexpr int kMaxPieces = 8;
    auto emit_packed = [&](int n, const int* pg, const int* r0, const int* cnt, int np, int g,
                           int slot, int kvh) -> bool {
      if (round >= 1) {
        const uint32_t par = (round - 1) & 1;
        uint64_t t_start = 0;
        while (!mbar_try_wait(&empty[ps], par)) {
          if (flags[0] != 0 || flags[1] != 0) return false;
          const uint64_t now = globaltimer();
          if (t_start == 0) t_start = now;
          else if (now - t_start > kWaitLimitNs) {
            dev_error(p.status, SKV_DEV_TIMEOUT);
            flags[1] = 1;
            aborted = true;
            return false;
          }
        }
      }
      meta[ps] = make_int4(n, g, slot, 0);
      unsigned char* sK = smem + ps * C::STAGE_BYTES;
      unsigned char* sV = sK + kTileBytes;
      mbar_arrive_expect_tx(&full[ps], (uint32_t)n * kRowBytes * 2);
      int row = 0;
      for (int i = 0; i < np; ++i) {
        const size_t src = ((size_t)pg[i] * p.Hkv + kvh) * head_stride + (size_t)r0[i] * kHeadDim;
        bulk_load(sK + row * kRowBytes, p.k_pool + src, (uint32_t)cnt[i] * kRowBytes, &full[ps], pol);
        bulk_load(sV + row * kRowBytes, p.v_pool + src, (uint32_t)cnt[i] * kRowBytes, &full[ps], pol);
        row += cnt[i];
      }
      ++e;
      if (++ps == ST) {
        ps = 0;
        ++round;
      }
      return true;
    };
    auto run_segments = [&](Trav& tr, int g, int slot, int kvh) -> bool {
      int pg[kMaxPieces], r0[kMaxPieces], cnt[kMaxPieces];
      int np = 0, rows = 0, tiles = 0;
      int page = 0, first = 0, c = 0;
      while (flags[0] == 0 && tr.next_piece(page, first, c, p.status)) {
        while (c > 0) {
          const int take = min(c, kBlock - rows);
          pg[np] = page;
          r0[np] = first;
          cnt[np] = take;
          ++np;
          rows += take;
          first += take;
          c -= take;
          if (rows == kBlock || np == kMaxPieces) {
            if (!emit_packed(rows, pg, r0, cnt, np, g, slot, kvh)) return false;
            ++tiles;
            np = rows = 0;
          }
        }
      }
      if (flags[0] != 0) return false;
      if (rows > 0) {
        if (!emit_packed(rows, pg, r0, cnt, np, g, slot, kvh)) return false;
        ++tiles;
      }
      if (tiles == 0 && !emit(0, g, slot, kvh, 0, 0, 0, 0)) return false;
      return true;
    };
    // All entries of one group segment; a segment without valid tiles still
    // issues a marker so that the consumers account for the group.
    auto run_group = [&](Trav& tr, int g, int slot, int kvh) -> bool {
      if (tr.mode == TRAV_SEGMENTS) return run_segments(tr, g, slot, kvh);
      int t0 = 0, n = 0, pg1 = 0, pg2 = 0, n1 = 0, cnt = 0;
      while (flags[0] == 0 && tr.next(t0, n, pg1, pg2, n1, p.status)) {
        if (!emit(n, g, slot, kvh, t0, pg1, pg2, n1)) return false;
        ++cnt;
      }
      if (flags[0] != 0) return false;
      if (cnt == 0 && !emit(0, g, slot, kvh, 0, 0, 0, 0)) return false;
      return true;
    };

    bool ok = true;
    if (!ART && p.sched == SCHED_PERSISTENT) {
      const int T = pre[p.B];
      const int P = p.n_ctas, c = blockIdx.x;
      int x = (int)(((long long)c * T) / P);
      const int hi = (int)(((long long)(c + 1) * T) / P);
      while (ok && x < hi) {
        int lo_b = 0, hi_b = p.B;  // largest b with pre[b] <= x
        while (hi_b - lo_b > 1) {
          const int mid = (lo_b + hi_b) >> 1;
          if (pre[mid] <= x) lo_b = mid; else hi_b = mid;
        }
        const int b = lo_b;
        const int nt = (pre[b + 1] - pre[b]) / p.Hkv;
        const int off = x - pre[b];
        const int kvh = off / nt, ti = off % nt;
        const int te = min(nt, ti + (hi - x));
        Trav tr;
        tr.init(p, false, b, kvh, Lsm[b], 0);
        tr.set_range(ti, te);
        const int g = b * p.Hkv + kvh;
        ok = run_group(tr, g, c + g, kvh);
        x += te - ti;
      }
    } else {
      const int split = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
      int L = p.seq_lens[b];
      if (L < 0 || L > p.max_seq_len) {
        if (split == 0 && kvh == 0) dev_error(p.status, SKV_DEV_BAD_SEQLEN);
        L = 0;
      }
      Trav tr;
      tr.init(p, ART, b, kvh, L, split);
      const int g = b * p.Hkv + kvh;
      ok = run_group(tr, g, g * p.n_splits + split, kvh);
    }
    if (ok) emit(-1, -1, 0, 0, 0, 0, 0, 0);
    // Copies the consumers never waited for (ART stop, abort) must land before
    // the CTA exits: learn how many entries they consumed, then drain the rest.
    const uint64_t t_start = globaltimer();
    while (flags[2] == 0 && globaltimer() - t_start < kWaitLimitNs) {
    }
    int consumed = flags[2] - 1;
    if (consumed < 0 || aborted || flags[1] != 0) consumed = 0;
    for (int kk = (e - ST > consumed ? e - ST : consumed); kk < e; ++kk)
      mbar_wait_bounded(&full[kk % ST], (kk / ST) & 1, nullptr);
    return;
  }

  // ------------------------------------------------------------------ consumers
  Warp<G, NW, ART, MINB> W;
  const int c = lane & 15, par = lane >> 4;
  const int Xl = ((lane & 15) >> (4 - C::S)) << (C::LN - C::S);
  const int Xg = Xl & (G - 1), Xi = Xl >> C::LG;
  const int rb = warp * C::RPW;
#pragma unroll
  for (int i = 0; i < C::STEPS; ++i) W.koff[i] = (rb + par + 2 * (i ^ Xi)) * kRowBytes + c * 16;
  W.voff = rb * kRowBytes + lane * 8;
#pragma unroll
  for (int j = 0; j < C::VPL; ++j) W.hd[j] = (Xl + j) & (G - 1);
  W.lrow = par + 2 * (Xl >> C::LG);
  W.owner = (lane & (16 | (C::STEPS == 4 ? 12 : 8))) == 0;

  auto reset_state = [&]() {
#pragma unroll
    for (int j = 0; j < C::VPL; ++j) {
      W.m_st[j] = -INFINITY;
      W.l_st[j] = 0.f;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) W.acc[g][0] = W.acc[g][1] = pack2(0.f, 0.f);
  };
  auto load_q = [&](int grp) {
    const int b = grp / p.Hkv, kvh = grp % p.Hkv;
    const uint16_t* qrow = p.q + ((size_t)b * p.Hq + (size_t)kvh * G) * kHeadDim + c * 8;
#pragma unroll
    for (int gr = 0; gr < G; ++gr) {
      const uint4 w = *reinterpret_cast<const uint4*>(qrow + (size_t)(gr ^ Xg) * kHeadDim);
      const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (int u = 0; u < 4; ++u)
        W.qf[gr][u] = pack2(__uint_as_float(ws[u] << 16) * p.qscale,
                            __uint_as_float(ws[u] & 0xFFFF0000u) * p.qscale);
    }
  };
  // Partial record of this warp for one (group piece): O (unnormalised),
  // m (base 2), l and the number of tiles folded.
  auto flush = [&](int slot, int tiles) {
    float* rec = p.ws_rec + ((size_t)slot * NW + warp) * G * kRecFloats;
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float x0, x1, x2, x3;
      unpack2(W.acc[g][0], x0, x1);
      unpack2(W.acc[g][1], x2, x3);
      *reinterpret_cast<float4*>(rec + g * kRecFloats + lane * 4) = make_float4(x0, x1, x2, x3);
    }
    if (W.owner) {
#pragma unroll
      for (int j = 0; j < C::VPL; ++j)
        *reinterpret_cast<float4*>(rec + W.hd[j] * kRecFloats + 128) =
            make_float4(W.m_st[j], W.l_st[j], (float)tiles, 0.f);
    }
  };

  float2* pbuf = reinterpret_cast<float2*>(smem + C::OFF_P) + warp * C::RPW * G;
  float2* abuf = reinterpret_cast<float2*>(smem + C::OFF_A) + warp * G;
  float* probe = reinterpret_cast<float*>(smem + C::OFF_PROBE);

  // ART state, identical in every consumer warp
  uint32_t done_mask = 0;
  int used[G];
#pragma unroll
  for (int g = 0; g < G; ++g) used[g] = 0;
  constexpr int SG = ART ? G : 1;
  float snapA_m[C::VPL], snapA_l[C::VPL], snapB_m[C::VPL], snapB_l[C::VPL];
  f2 snapA_acc[SG][2], snapB_acc[SG][2];
#pragma unroll
  for (int j = 0; j < C::VPL; ++j) snapA_m[j] = snapA_l[j] = snapB_m[j] = snapB_l[j] = 0.f;
#pragma unroll
  for (int g = 0; g < SG; ++g)
    snapA_acc[g][0] = snapA_acc[g][1] = snapB_acc[g][0] = snapB_acc[g][1] = pack2(0.f, 0.f);
  // judge state (warps < G judge head `warp`)
  constexpr int DGR = 32 / NW, DPG = 8 / DGR;
  float jx_prev[DPG];
#pragma unroll
  for (int d = 0; d < DPG; ++d) jx_prev[d] = 0.f;
  int j_cnt = 0;
  bool j_done = false;

  // Apply the decisions for tile t (all heads): restore a head that stops
  // after tile t from snapshot A (= state after tile t).
  auto art_apply = [&](int t) -> bool {
    if (!mbar_wait_bounded(&dec_bar[t % 3], (t / 3) & 1, &flags[1])) {
      if (lane == 0) {
        dev_error(p.status, SKV_DEV_TIMEOUT);
        flags[1] = 1;
      }
      return false;
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      if (((done_mask >> g) & 1u) == 0 && dec[(t % 3) * G + g] != 0) {
        done_mask |= 1u << g;
        used[g] = t + 1;
        W.acc[g][0] = snapA_acc[g][0];
        W.acc[g][1] = snapA_acc[g][1];
#pragma unroll
        for (int j = 0; j < C::VPL; ++j)
          if (W.hd[j] == g) {
            W.m_st[j] = snapA_m[j];
            W.l_st[j] = snapA_l[j];
          }
      }
    }
    return true;
  };

  // Judge warp `warp`: probe of head `warp` after tile t and the stopping rule.
  auto art_judge = [&](int t) -> bool {
    const int g = warp;
    if (!mbar_wait_bounded(&probe_bar[t % 3], (t / 3) & 1, &flags[1])) {
      if (lane == 0) {
        dev_error(p.status, SKV_DEV_TIMEOUT);
        flags[1] = 1;
      }
      return false;
    }
    const int src = lane % NW, dg = lane / NW;
    const float* pe = probe + ((size_t)(t % 3) * NW + src) * G * C::PROBE + g * C::PROBE;
    const float mw = pe[0];
    float M = mw;
#pragma unroll
    for (int m = 1; m < NW; m <<= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, m));
    const float f = (M == -INFINITY) ? 0.f : exp2f(mw - M);
    float Ls = pe[1] * f;
    float X[DPG];
#pragma unroll
    for (int d = 0; d < DPG; ++d) X[d] = pe[4 + dg * DPG + d] * f;
#pragma unroll
    for (int m = 1; m < NW; m <<= 1) {
      Ls += __shfl_xor_sync(0xffffffffu, Ls, m);
#pragma unroll
      for (int d = 0; d < DPG; ++d) X[d] += __shfl_xor_sync(0xffffffffu, X[d], m);
    }
    float nx = 0.f, np = 0.f;
#pragma unroll
    for (int d = 0; d < DPG; ++d) {
      X[d] = (Ls > 0.f) ? X[d] / Ls : 0.f;
      nx += X[d] * X[d];
      np += jx_prev[d] * jx_prev[d];
    }
#pragma unroll
    for (int m = NW; m < 32; m <<= 1) {
      nx += __shfl_xor_sync(0xffffffffu, nx, m);
      np += __shfl_xor_sync(0xffffffffu, np, m);
    }
    const float a = sqrtf(nx), bp = sqrtf(np);
    float dd = 0.f;
#pragma unroll
    for (int d = 0; d < DPG; ++d) {
      const float du = ((a > 0.f) ? X[d] / a : 0.f) - ((bp > 0.f) ? jx_prev[d] / bp : 0.f);
      dd += du * du;
      jx_prev[d] = X[d];
    }
#pragma unroll
    for (int m = NW; m < 32; m <<= 1) dd += __shfl_xor_sync(0xffffffffu, dd, m);
    float d_s, d_c;
    if (bp == 0.f) d_s = (a == 0.f) ? 0.f : INFINITY;
    else d_s = fabsf(a - bp) / bp;
    if (a == 0.f || bp == 0.f) d_c = (a == 0.f && bp == 0.f) ? 0.f : 1.f;
    else d_c = 0.5f * dd;  // 1 - cos(x, x') = |x/|x| - x'/|x'||^2 / 2
    int stop = 0;
    if (!j_done) {
      const bool pass = (t >= 1) && (d_s < p.tau) && (d_c < p.phi);
      j_cnt = pass ? j_cnt + 1 : 0;
      if (j_cnt >= p.patience) {
        stop = 1;
        j_done = true;
      }
    }
    if (lane == 0) dec[(t % 3) * G + g] = stop;
    __syncwarp();
    mbar_arrive_if(&dec_bar[t % 3], lane == 0);
    return true;
  };

  int e = 0, s = 0;       // ring entries consumed, stage
  uint32_t ph = 0;        // phase of the current ring round
  int k = 0;              // tiles folded for the current group (ART: tile index)
  int cur_g = -1, cur_slot = 0;
  bool all_stopped = false;
  reset_state();
  while (true) {
    if (!mbar_wait_bounded(&full[s], ph, &flags[1])) {
      if (lane == 0) {
        dev_error(p.status, SKV_DEV_TIMEOUT);
        flags[1] = 1;
      }
      break;
    }
    const int4 mt = meta[s];
    const int n = mt.x;
    if (n < 0) break;  // end of traversal
    if (mt.y != cur_g) {
      if (!ART && cur_g >= 0) flush(cur_slot, k);
      reset_state();
      load_q(mt.y);
      cur_g = mt.y;
      cur_slot = mt.z;
      k = 0;
    }
    if (n > 0) {
      const unsigned char* sK = smem + s * C::STAGE_BYTES;
      const unsigned char* sV = sK + kTileBytes;
      const int nv = n - rb;
      if (nv >= C::RPW) fold_tile<G, NW, ART, MINB, false>(W, sK, sV, nv, done_mask, pbuf, abuf);
      else fold_tile<G, NW, ART, MINB, true>(W, sK, sV, nv, done_mask, pbuf, abuf);
    }
    mbar_arrive_if(&empty[s], lane == 0);
    ++e;
    if (++s == ST) {
      s = 0;
      ph ^= 1u;
    }
    if (n == 0) continue;

    if constexpr (ART) {
      // Tile k has been folded.  (1) publish (m, l, O[0:8]) per head for tile
      // k; (2) apply the decisions for tile k-2, restoring heads that stop
      // there from the snapshot taken after tile k-2; (3) rotate snapshots;
      // (4) judge warps decide tile k-1, whose records are complete by now.
      float* pw = probe + ((size_t)(k % 3) * NW + warp) * G * C::PROBE;
      if (W.owner) {
#pragma unroll
        for (int j = 0; j < C::VPL; ++j) {
          pw[W.hd[j] * C::PROBE + 0] = W.m_st[j];
          pw[W.hd[j] * C::PROBE + 1] = W.l_st[j];
        }
      }
      if (lane < 2) {
#pragma unroll
        for (int g = 0; g < G; ++g) {
          float x0, x1, x2, x3;
          unpack2(W.acc[g][0], x0, x1);
          unpack2(W.acc[g][1], x2, x3);
          *reinterpret_cast<float4*>(pw + g * C::PROBE + 4 + lane * 4) = make_float4(x0, x1, x2, x3);
        }
      }
      __syncwarp();
      mbar_arrive_if(&probe_bar[k % 3], lane == 0);

      if (k >= 2) {
        if (!art_apply(k - 2)) break;
        if (done_mask == (1u << G) - 1u) {
          if (warp == 0 && lane == 0) flags[0] = e + 1;  // entries consumed + 1
          ++k;
          all_stopped = true;
          break;
        }
      }
      // snapshots: A <- state after tile k-1, B <- state after tile k
#pragma unroll
      for (int j = 0; j < C::VPL; ++j) {
        snapA_m[j] = snapB_m[j];
        snapA_l[j] = snapB_l[j];
        snapB_m[j] = W.m_st[j];
        snapB_l[j] = W.l_st[j];
      }
#pragma unroll
      for (int g = 0; g < G; ++g) {
        snapA_acc[g][0] = snapB_acc[g][0];
        snapA_acc[g][1] = snapB_acc[g][1];
        snapB_acc[g][0] = W.acc[g][0];
        snapB_acc[g][1] = W.acc[g][1];
      }
      if (warp < G && k >= 1) {
        if (!art_judge(k - 1)) break;
      }
    }
    ++k;
  }
  if constexpr (ART) {
    // end of the traversal: the decision for the second-to-last tile is still
    // pending (a stop after the last tile changes nothing)
    if (!all_stopped && flags[1] == 0 && k >= 2) art_apply(k - 2);
  }

  // ------------------------------------------------------------------ epilogue
  if constexpr (!ART) {
    if (cur_g >= 0) flush(cur_slot, k);
    // Every consumer warp ends here: let the producer know once all are done.
    __syncwarp();
    mbar_arrive_if(fin_bar, lane == 0);
    if (warp == 0) {
      if (!mbar_wait_bounded(fin_bar, 0, nullptr) && lane == 0) dev_error(p.status, SKV_DEV_TIMEOUT);
      if (lane == 0) flags[2] = (flags[1] != 0) ? 1 : e + 1;
    }
    return;
  } else {
    float* fin = reinterpret_cast<float*>(smem + C::OFF_FIN);
    float2* finml = reinterpret_cast<float2*>(smem + C::OFF_FINML);
    if (W.owner) {
#pragma unroll
      for (int j = 0; j < C::VPL; ++j) finml[warp * G + W.hd[j]] = make_float2(W.m_st[j], W.l_st[j]);
    }
#pragma unroll
    for (int g = 0; g < G; ++g) {
      float x0, x1, x2, x3;
      unpack2(W.acc[g][0], x0, x1);
      unpack2(W.acc[g][1], x2, x3);
      *reinterpret_cast<float4*>(fin + (warp * G + g) * kHeadDim + lane * 4) = make_float4(x0, x1, x2, x3);
    }
    __syncwarp();
    mbar_arrive_if(fin_bar, lane == 0);
    if (!mbar_wait_bounded(fin_bar, 0, nullptr)) {
      if (lane == 0) dev_error(p.status, SKV_DEV_TIMEOUT);
    }
    if (threadIdx.x == 0) flags[2] = (flags[1] != 0) ? 1 : e + 1;
    const int b = blockIdx.z, h0 = blockIdx.y * G;
    for (int o = threadIdx.x; o < G * kHeadDim; o += NW * 32) {
      const int g = o / kHeadDim, dim = o % kHeadDim;
      float M = -INFINITY;
#pragma unroll
      for (int w = 0; w < NW; ++w) M = fmaxf(M, finml[w * G + g].x);
      float Ls = 0.f, X = 0.f;
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          const float2 ml = finml[w * G + g];
          const float f = exp2f(ml.x - M);
          Ls += ml.y * f;
          X += fin[(w * G + g) * kHeadDim + dim] * f;
        }
      }
      const size_t row = (size_t)b * p.Hq + h0 + g;
      p.out[row * kHeadDim + dim] = (Ls > 0.f) ? X / Ls : 0.f;
      if (dim == 0) {
        p.lse[row] = (Ls > 0.f) ? (M + log2f(Ls)) * kLn2 : -INFINITY;
        if (p.blocks_consumed) {
          int u = k;
#pragma unroll
          for (int gg = 0; gg < G; ++gg)
            if (gg == g && ((done_mask >> gg) & 1u)) u = used[gg];
          p.blocks_consumed[row] = u;
        }
      }
    }
  }
}

template <int G, bool ART>
constexpr int nw_for() {
  return (ART || G == 8) ? SKV_CONSUMER_WARPS_ART : SKV_CONSUMER_WARPS;
}
template <int G, bool ART>
constexpr int minb_for() {
  return (ART || G == 8) ? 1 : SKV_CTAS_PER_SM;
}

template <int G, bool ART>
int launch_t(const DecodeParams& p, cudaStream_t st) {
  constexpr int NW = nw_for<G, ART>();
  constexpr int MINB = minb_for<G, ART>();
  using C = Cfg<G, NW, ART, MINB>;
  auto kern = decode_kernel<G, ART, NW, MINB>;
  // Set the shared-memory attribute once per device (not inside a capture).
  static bool attr_set[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return (int)cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::TOTAL);
    if (err != cudaSuccess) return (int)err;
    attr_set[dev] = true;
  }
  dim3 grid;
  if (!ART && p.sched == SCHED_PERSISTENT) grid = dim3(p.n_ctas, 1, 1);
  else grid = dim3(ART ? 1 : p.n_splits, p.Hkv, p.B);
  kern<<<grid, C::THREADS, C::TOTAL, st>>>(p);
  return (int)cudaGetLastError();
}

}  // namespace

int decode_consumer_warps(int G, bool art) {
  switch (G) {
    case 1: return art ? nw_for<1, true>() : nw_for<1, false>();
    case 2: return art ? nw_for<2, true>() : nw_for<2, false>();
    case 4: return art ? nw_for<4, true>() : nw_for<4, false>();
    default: return art ? nw_for<8, true>() : nw_for<8, false>();
  }
}

int decode_ctas_per_sm(int G, bool art) {
  switch (G) {
    case 1: return art ? minb_for<1, true>() : minb_for<1, false>();
    case 2: return art ? minb_for<2, true>() : minb_for<2, false>();
    case 4: return art ? minb_for<4, true>() : minb_for<4, false>();
    default: return art ? minb_for<8, true>() : minb_for<8, false>();
  }
}

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
