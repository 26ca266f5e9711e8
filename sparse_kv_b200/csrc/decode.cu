// decode.cu -- streaming block-wise decode attention for sm_100a (plain
// traversals: whole sequence, token range, sink + recent window, caller's
// block order, caller's token segments).  Run-time termination (ART) has its
// own kernel in art.cu.
//
// Structure of a CTA: the last warp is the producer.  One of its lanes walks
// the traversal and issues bulk-async copies (TMA engine, cp.async.bulk, no
// multicast) of the K and V rows of each tile (<= 64 consecutive tokens from
// <= 2 pages) into a STAGES-deep shared-memory ring guarded by full/empty
// mbarriers, publishing each entry's row count and KV group in shared memory.
// NW consumer warps split every tile's 64 rows (64/NW each) and keep their own
// online-softmax state (m, l, O) for the G query heads of the group (the warp
// arithmetic is in tile.cuh).
//
// Schedules.  Index-based traversals run persistently: one CTA per SM takes
// an even share of the concatenated tile lists of all KV groups (a share may
// span group boundaries; consumers then write a partial record per warp and
// start the next group without any CTA-wide synchronisation).  Segment lists
// split each group across a fixed number of CTAs.  Both end with an exact
// merge of the per-warp records (launch_merge_records).
#include "common.cuh"
#include "decode.cuh"
#include "tile.cuh"

// SKV_CONSUMER_WARPS consumer warps per CTA and SKV_CTAS_PER_SM resident CTAs
// per SM (both CTAs' warps hide each other's latency; fewer warps per tile
// means fewer per-warp fixed costs).  8-head groups use 8 warps and one CTA
// per SM (their state needs registers).
#ifndef SKV_CONSUMER_WARPS
#define SKV_CONSUMER_WARPS 8
#endif
#ifndef SKV_CTAS_PER_SM
#define SKV_CTAS_PER_SM 2
#endif

namespace skv {
namespace {

// ---------------------------------------------------------------------------
// Traversal: yields tiles (t0, n) = n <= 64 consecutive tokens from t0, with
// the page(s) holding them.
// ---------------------------------------------------------------------------
struct Trav {
  int mode, L, nb;
  const int* bt;  // block_table row of this sequence
  int num_pages;
  // index-based modes
  int i, i_end;
  int ra, re;      // natural / range token interval
  int A, Rs, nt1;  // window: [0, A) then [Rs, L)
  const int* ord;
  // segments
  const int* ss;
  const int* se;
  int seg_i, seg_end_i;  // (walked by the producer warp, run_segments_warp)

  // Whole traversal of group (b, kvh), then narrowed with set_range
  // (index-based modes: tile indices; segments: segment indices).
  __device__ void init(const DecodeParams& p, int b, int kvh, int L_, int split) {
    mode = p.mode;
    L = L_;
    nb = (L + kBlock - 1) / kBlock;
    bt = p.block_table + (size_t)b * p.max_blocks;
    num_pages = p.num_pages;
    ord = nullptr;
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
    const int S = p.n_splits > 0 ? p.n_splits : 1;
    set_range((int)(((long long)split * N) / S), (int)(((long long)(split + 1) * N) / S));
  }

  __device__ void set_range(int lo, int hi) {
    if (mode == TRAV_SEGMENTS) {
      seg_i = lo;
      seg_end_i = hi;
    } else {
      i = lo;
      i_end = hi;
    }
  }

  // Index-based modes (segment lists take the split schedule, whose producer
  // warp packs them: run_segments_warp).
  __device__ bool next(int& t0, int& n, int& pg1, int& pg2, int& n1, uint32_t* status) {
    while (true) {
      int a, e;
      if (mode == TRAV_ORDER) {
        if (i >= i_end) return false;
        const int j = ord[i++];
        if (j < 0 || j >= nb) {
          dev_error(status, SKV_DEV_BAD_ORDER);
          continue;
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

// ---- thread-block cluster helpers (the split schedule: a cluster = the pieces of one group)
__device__ __forceinline__ uint32_t cluster_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
// Arrive on an mbarrier of another CTA of the cluster (release: this thread's
// and, after the fence, its CTA's earlier shared-memory writes are visible).
__device__ __forceinline__ void cluster_arrive_remote(uint32_t bar_cluster_addr) {
  asm volatile("fence.acq_rel.cluster;\n\tmbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];"
               ::"r"(bar_cluster_addr) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait_cluster(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait (acquire at cluster scope): gives up after `limit_ns`.
__device__ __forceinline__ bool mbar_wait_cluster(uint64_t* bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  while (true) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if (globaltimer() - t0 > limit_ns) return false;
  }
}
__device__ __forceinline__ float4 ld_cluster_f4(uint32_t addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(addr)
               : "memory");
  return v;
}

template <int G, int NW, int MINB>
struct Cfg {
  using Ln = Lanes<G, NW>;
  static constexpr int RPW = Ln::RPW;
  static constexpr int STAGES = MINB == 2 ? 3 : 6;
  static constexpr int THREADS = (NW + 1) * 32;
  static constexpr size_t STAGE_BYTES = 2 * (size_t)kTileBytes;
  static constexpr int NBAR = 2 * STAGES + 6;  // full, empty, fin, fin2, fin3, fin4, gather, release
  static constexpr size_t OFF_BAR = STAGES * STAGE_BYTES;
  static constexpr size_t OFF_META = (OFF_BAR + NBAR * 8 + 15) / 16 * 16;   // int4 [STAGES]
  static constexpr size_t OFF_FLAGS = (OFF_META + STAGES * 16 + 15) / 16 * 16;
  static constexpr size_t OFF_P = OFF_FLAGS + 16;                         // float2 [NW][RPW][G]
  static constexpr size_t OFF_A = OFF_P + (size_t)NW * RPW * G * 8;        // float2 [NW][G]
  static constexpr size_t OFF_PRE = OFF_A + (size_t)NW * G * 8;            // int [B+1], int [B]
  static constexpr size_t N_PRE = (2 * (size_t)kMaxPersistentBatch + 1) * 4;
  static constexpr size_t TOTAL = OFF_PRE + N_PRE;
  static_assert(TOTAL <= (MINB == 2 ? 113 : 227) * 1024, "shared memory budget");
  // every region read or written with 16-byte vectors starts 16-byte aligned
  static_assert(OFF_BAR % 16 == 0 && OFF_META % 16 == 0 && OFF_FLAGS % 16 == 0, "alignment");
  static_assert(OFF_P % 16 == 0 && OFF_A % 16 == 0 && OFF_PRE % 16 == 0, "alignment");
  static_assert((RPW * G * 8) % 16 == 0 || G == 1, "pbuf rows");
  static_assert((kRecFloats * 4) % 16 == 0, "record strides");
};

template <int G, int NW, int MINB>
__global__ void __launch_bounds__(Cfg<G, NW, MINB>::THREADS, MINB) decode_kernel(const DecodeParams p) {
  using C = Cfg<G, NW, MINB>;
  constexpr int ST = C::STAGES;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + ST;
  uint64_t* fin_bar = empty + ST;  // NW arrivals: the consumers are done with the ring
  // split schedule only:
  uint64_t* fin2_bar = fin_bar + 1;     // NW arrivals: the warps' states are in the ring
  uint64_t* fin3_bar = fin2_bar + 1;    // NW arrivals: the piece's records are written
  uint64_t* fin4_bar = fin3_bar + 1;    // G arrivals: (rank 0) the merge is done
  uint64_t* gather_bar = fin4_bar + 1;  // (rank 0) S arrivals, one per piece of the cluster
  uint64_t* release_bar = gather_bar + 1;  // (ranks > 0) rank 0 has read this CTA's records
  int4* meta = reinterpret_cast<int4*>(smem + C::OFF_META);  // {rows, group, slot, 0}
  volatile int* flags = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  // flags[1]: abort (a bounded wait expired)
  // flags[2]: consumers finished (entries consumed + 1; 0 = running)

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NW);
    }
    mbar_init(fin_bar, NW);
    mbar_init(fin2_bar, NW);
    mbar_init(fin3_bar, NW);
    mbar_init(fin4_bar, G);
    mbar_init(gather_bar, p.sched == SCHED_SPLIT ? p.n_splits : 1);
    mbar_init(release_bar, 1);
    flags[0] = flags[1] = flags[2] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  // Split schedule: every thread marks the cluster barrier once its CTA's
  // mbarriers are initialised (release); a wait on it before the first access
  // to another CTA's shared memory then ends as soon as every CTA of the
  // cluster is running with its barriers ready.
  if (p.sched == SCHED_SPLIT) asm volatile("barrier.cluster.arrive.aligned;" ::: "memory");
  // ------------------------------------------------------------------ producer
  if (warp == NW) {
    int* pre = reinterpret_cast<int*>(smem + C::OFF_PRE);  // [B+1] tiles before batch b
    int* Lsm = pre + kMaxPersistentBatch + 1;              // [B] validated lengths
    if (p.sched == SCHED_PERSISTENT) {
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
    // Segment lists on the split schedule keep the whole warp: it resolves
    // segments 32 at a time (below); elsewhere lane 0 alone produces.
    const bool warp_segments = p.sched == SCHED_SPLIT && p.mode == TRAV_SEGMENTS;
    if (!warp_segments && lane != 0) return;

    const uint64_t pol = policy_evict_first();
    const size_t head_stride = (size_t)kBlock * kHeadDim;
    int e = 0, ps = 0, round = 0;  // entries issued, stage, ring round
    bool aborted = false;
    // test hook: this CTA stops issuing before entry `withhold` (-1: never)
    const int cta = (int)(blockIdx.x + gridDim.x * (blockIdx.y + gridDim.y * blockIdx.z));
    const int withhold = (p.withhold_entry > 0 && cta == p.withhold_cta) ? p.withhold_entry - 1 : -1;
    // Issue one ring entry: `n` rows of group `g` (n = 0: a group marker with
    // no rows, n = -1: end of traversal).  Returns false to stop issuing.
    auto emit = [&](int n, int g, int slot, int kvh, int t0, int pg1, int pg2, int n1) -> bool {
      if (e == withhold) return false;  // nothing issued: the consumers' wait expires
      if (round >= 1) {
        const uint32_t par = (round - 1) & 1;
        uint64_t t_start = 0;
        while (!mbar_try_wait(&empty[ps], par)) {
          if (flags[1] != 0) return false;
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
    constexpr int kMaxPieces = 8;  // bulk copies (pieces) packed into one ring entry
    auto emit_packed = [&](int n, const int* pg, const int* r0, const int* cnt, int np, int g,
                           int slot, int kvh) -> bool {
      if (e == withhold) return false;
      if (round >= 1) {
        const uint32_t par = (round - 1) & 1;
        uint64_t t_start = 0;
        while (!mbar_try_wait(&empty[ps], par)) {
          if (flags[1] != 0) return false;
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
    // Segment lists: rows of several segments are packed into full 64-row
    // tiles (attention over a key set does not depend on the keys' order),
    // one bulk copy per piece (<= 64 consecutive tokens of one page).  The
    // segments are resolved by the whole warp, 32 at a time: lane i loads segment i's bounds and the pages of its first two
    // blocks (independent loads, one round trip for the batch) into shared
    // memory, and lane 0 then issues the copies without waiting on global
    // memory (a segment reaching past two blocks loads its further pages as it
    // goes).  Called by every lane; returns lane 0's verdict on all lanes.
    auto run_segments_warp = [&](Trav& tr, int g, int slot, int kvh) -> bool {
      int4* stage = reinterpret_cast<int4*>(smem + C::OFF_PRE);  // [32] {start, stop, page0, page1}
      int pg[kMaxPieces], r0[kMaxPieces], cnt[kMaxPieces];
      int np = 0, rows = 0, tiles = 0;
      bool good = true;
      for (int base = tr.seg_i; base < tr.seg_end_i; base += 32) {
        const int i = base + lane;
        int4 v = make_int4(0, 0, -1, -1);
        if (i < tr.seg_end_i) {
          int a = tr.ss[i], t = tr.se[i];
          if (a > t) {
            dev_error(p.status, SKV_DEV_BAD_SEGMENT);
            a = t = 0;
          }
          a = max(a, 0);
          t = min(t, tr.L);
          if (t > a) {
            const int b0 = a / kBlock;
            int p0 = tr.bt[b0], p1 = -1;
            if ((t - 1) / kBlock > b0) p1 = tr.bt[b0 + 1];
            if (p0 < 0 || p0 >= tr.num_pages) {
              dev_error(p.status, SKV_DEV_BAD_PAGE);
              p0 = -1;
            }
            if ((t - 1) / kBlock > b0 && (p1 < 0 || p1 >= tr.num_pages)) {
              dev_error(p.status, SKV_DEV_BAD_PAGE);
              p1 = -1;
            }
            v = make_int4(a, t, p0, p1);
          }
        }
        __syncwarp();  // lane 0 is done with the previous batch
        stage[lane] = v;
        __syncwarp();
        if (lane == 0) {
          const int nseg = min(32, tr.seg_end_i - base);
          for (int k2 = 0; k2 < nseg && good; ++k2) {
            const int4 sv = stage[k2];
            const int b0 = sv.x / kBlock;
            for (int pos = sv.x; pos < sv.y && good;) {
              const int blk = pos / kBlock, first = pos % kBlock;
              const int c = min(kBlock - first, sv.y - pos);
              pos += c;
              int page = blk == b0 ? sv.z : blk == b0 + 1 ? sv.w : tr.bt[blk];
              if (blk > b0 + 1 && (page < 0 || page >= tr.num_pages)) {
                dev_error(p.status, SKV_DEV_BAD_PAGE);
                page = -1;
              }
              if (page < 0) continue;  // (flagged)
              for (int f = first, left = c; left > 0;) {
                const int take = min(left, kBlock - rows);
                pg[np] = page;
                r0[np] = f;
                cnt[np] = take;
                ++np;
                rows += take;
                f += take;
                left -= take;
                if (rows == kBlock || np == kMaxPieces) {
                  if (!emit_packed(rows, pg, r0, cnt, np, g, slot, kvh)) {
                    good = false;
                    break;
                  }
                  ++tiles;
                  np = rows = 0;
                }
              }
            }
          }
        }
        if (!__shfl_sync(0xffffffffu, good, 0)) return false;
      }
      if (lane == 0) {
        if (rows > 0) {
          if (emit_packed(rows, pg, r0, cnt, np, g, slot, kvh)) ++tiles;
          else good = false;
        }
        if (good && tiles == 0 && !emit(0, g, slot, kvh, 0, 0, 0, 0)) good = false;
      }
      return __shfl_sync(0xffffffffu, good, 0);
    };
    // All entries of one group segment; a segment without valid tiles still
    // issues a marker so that the consumers account for the group.
    auto run_group = [&](Trav& tr, int g, int slot, int kvh) -> bool {
      int t0 = 0, n = 0, pg1 = 0, pg2 = 0, n1 = 0, cnt = 0;
      while (tr.next(t0, n, pg1, pg2, n1, p.status)) {
        if (!emit(n, g, slot, kvh, t0, pg1, pg2, n1)) return false;
        ++cnt;
      }
      if (cnt == 0 && !emit(0, g, slot, kvh, 0, 0, 0, 0)) return false;
      return true;
    };

    bool ok = true;
    if (p.sched == SCHED_PERSISTENT) {
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
        tr.init(p, b, kvh, Lsm[b], 0);
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
      tr.init(p, b, kvh, L, split);
      const int g = b * p.Hkv + kvh;
      if (warp_segments) {
        ok = run_segments_warp(tr, g, g * p.n_splits + split, kvh);
        if (lane != 0) return;
      } else {
        ok = run_group(tr, g, g * p.n_splits + split, kvh);
      }
    }
    if (ok) emit(-1, -1, 0, 0, 0, 0, 0, 0);
    // Copies the consumers never waited for (abort) must land before the CTA
    // exits: learn how many entries they consumed, then drain the rest.
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
  Warp<G, NW> W;
  W.setup(warp, lane);
  const int rb = warp * C::RPW;
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
      for (int j = 0; j < Lanes<G, NW>::VPL; ++j)
        *reinterpret_cast<float4*>(rec + W.hd[j] * kRecFloats + 128) =
            make_float4(W.m_st[j], W.l_st[j], (float)tiles, 0.f);
    }
  };

  float2* pbuf = reinterpret_cast<float2*>(smem + C::OFF_P) + warp * C::RPW * G;
  float2* abuf = reinterpret_cast<float2*>(smem + C::OFF_A) + warp * G;

  int e = 0, s = 0;       // ring entries consumed, stage
  uint32_t ph = 0;        // phase of the current ring round
  int k = 0;              // tiles folded for the current group piece
  int cur_g = -1, cur_slot = 0;
  bool saw_end = false;  // the end entry was reached: every copy into the ring has landed
  W.reset();
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
    if (n < 0) {  // end of traversal
      saw_end = true;
      break;
    }
    if (mt.y != cur_g) {
      if (cur_g >= 0) flush(cur_slot, k);
      W.reset();
      const int b = mt.y / p.Hkv, kvh = mt.y % p.Hkv;
      W.load_q(p.q, (size_t)b * p.Hq + (size_t)kvh * G, p.qscale, lane);
      cur_g = mt.y;
      cur_slot = mt.z;
      k = 0;
    }
    if (n > 0) {
      const unsigned char* sK = smem + s * C::STAGE_BYTES;
      const unsigned char* sV = sK + kTileBytes;
      const int nv = n - rb;
      if (nv >= C::RPW) fold_tile<G, NW, false>(W, sK, sV, nv, 0u, pbuf, abuf);
      else fold_tile<G, NW, true>(W, sK, sV, nv, 0u, pbuf, abuf);
    }
    mbar_arrive_if(&empty[s], lane == 0);
    ++e;
    if (++s == ST) {
      s = 0;
      ph ^= 1u;
    }
    if (n > 0) ++k;
  }

  // ------------------------------------------------------------------ epilogue
  if (p.sched == SCHED_PERSISTENT) {
    if (cur_g >= 0) flush(cur_slot, k);
    // Every consumer warp ends here: let the producer know once all are done.
    __syncwarp();
    mbar_arrive_if(fin_bar, lane == 0);
    if (warp == 0) {
      if (!mbar_wait_bounded(fin_bar, 0, nullptr) && lane == 0) dev_error(p.status, SKV_DEV_TIMEOUT);
      if (lane == 0) flags[2] = (flags[1] != 0) ? 1 : e + 1;
    }
    return;
  }
  // Split schedule: the CTAs of a cluster are the S pieces of one group, and
  // the merge happens here, over distributed shared memory.  Once every
  // consumer warp is done with the ring (no copy is in flight after the end
  // entry), the warps leave their states in it and warps 0..G-1 combine one
  // head each into this piece's record (also in shared memory).  Every CTA then
  // arrives on rank 0's gather barrier; rank 0 reads the S records of each head
  // from the cluster's shared memory, writes the output row and releases the
  // other CTAs, which stay resident until then.  Every wait is bounded; a CTA
  // whose walk failed sends an empty record (the status word has the error).
  __syncwarp();
  mbar_arrive_if(fin_bar, lane == 0);
  const bool fin_ok = mbar_wait_bounded(fin_bar, 0, nullptr);
  if (warp == 0 && lane == 0) {
    if (!fin_ok) dev_error(p.status, SKV_DEV_TIMEOUT);
    flags[2] = (flags[1] != 0) ? 1 : e + 1;
  }
  // after an abort a warp may have left the loop early (and copies may still land)
  const bool good = fin_ok && flags[1] == 0 && saw_end;
  float* st_sm = reinterpret_cast<float*>(smem);   // [NW][G][kRecFloats]: O, m, l, tiles
  float* pc_sm = st_sm + NW * G * kRecFloats;       // [G][kRecFloats]: this piece's records
  static_assert((size_t)(NW + 1) * G * kRecFloats * 4 <= ST * C::STAGE_BYTES, "states fit in the ring");
  if (good) {
#pragma unroll
    for (int g2 = 0; g2 < G; ++g2) {
      float x0, x1, x2, x3;
      unpack2(W.acc[g2][0], x0, x1);
      unpack2(W.acc[g2][1], x2, x3);
      *reinterpret_cast<float4*>(st_sm + (warp * G + g2) * kRecFloats + lane * 4) =
          make_float4(x0, x1, x2, x3);
    }
    if (W.owner) {
#pragma unroll
      for (int j = 0; j < Lanes<G, NW>::VPL; ++j)
        *reinterpret_cast<float4*>(st_sm + (warp * G + W.hd[j]) * kRecFloats + 128) =
            make_float4(W.m_st[j], W.l_st[j], (float)k, 0.f);
    }
  }
  __syncwarp();
  mbar_arrive_if(fin2_bar, lane == 0);
  const bool ok2 = mbar_wait_bounded(fin2_bar, 0, nullptr);
  if (warp < G) {  // this piece's record of head `warp`
    const int h = warp;
    float M = -INFINITY, L = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    if (good && ok2) {
#pragma unroll
      for (int w = 0; w < NW; ++w) {
        const float2 ml = *reinterpret_cast<const float2*>(st_sm + (w * G + h) * kRecFloats + 128);
        if (ml.y > 0.f) M = fmaxf(M, ml.x);
      }
      if (M != -INFINITY) {
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          const float* s = st_sm + (w * G + h) * kRecFloats;
          const float2 ml = *reinterpret_cast<const float2*>(s + 128);
          const float f = (ml.y > 0.f) ? exp2f(ml.x - M) : 0.f;
          const float4 x = *reinterpret_cast<const float4*>(s + lane * 4);
          L += ml.y * f;
          o.x += x.x * f;
          o.y += x.y * f;
          o.z += x.z * f;
          o.w += x.w * f;
        }
      }
    }
    *reinterpret_cast<float4*>(pc_sm + h * kRecFloats + lane * 4) = o;
    if (lane == 0)
      *reinterpret_cast<float4*>(pc_sm + h * kRecFloats + 128) =
          make_float4(M, L, (good && ok2) ? (float)k : 0.f, 0.f);
  }
  __syncwarp();
  mbar_arrive_if(fin3_bar, lane == 0);
  const bool ok3 = mbar_wait_bounded(fin3_bar, 0, nullptr);
  if (!ok2 || !ok3) {
    if (lane == 0) dev_error(p.status, SKV_DEV_TIMEOUT);
  }
  const uint32_t rank = blockIdx.x;  // cluster (S, 1, 1) over grid.x = S
  const int S = p.n_splits;
  if (warp == 0) {  // this piece is ready: tell rank 0
    asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
    if (lane == 0) cluster_arrive_remote(cluster_addr(gather_bar, 0));
  }
  if (rank == 0) {
    if (warp < G) {
      if (warp != 0) asm volatile("barrier.cluster.wait.aligned;" ::: "memory");
      const int h = warp;
      // (longer than any CTA's own bounded waits: a piece arrives once its walk ends)
      const bool got = mbar_wait_cluster(gather_bar, 0, 4 * kWaitLimitNs);
      if (!got && lane == 0) dev_error(p.status, SKV_DEV_TIMEOUT);
      if (got) {
        // lane s holds piece s's scalars (S <= 32)
        float ms = -INFINITY, ls = 0.f;
        int ts = 0;
        if (lane < S) {
          const float4 v = ld_cluster_f4(cluster_addr(pc_sm + h * kRecFloats + 128, lane));
          if (v.y > 0.f) {
            ms = v.x;
            ls = v.y;
          }
          ts = (int)v.z;
        }
        float M = ms;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) {
          M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
          ts += __shfl_xor_sync(0xffffffffu, ts, o);
        }
        const float fs = (ms != -INFINITY) ? exp2f(ms - M) : 0.f;
        float Wl = fs * ls;
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) Wl += __shfl_xor_sync(0xffffffffu, Wl, o);
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
        const uint32_t own = smem_u32(pc_sm + h * kRecFloats + lane * 4);
        for (int s0 = 0; s0 < S; s0 += 8) {
          float4 x[8];
          float f[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const int s = s0 + q;
            f[q] = __shfl_sync(0xffffffffu, fs, s & 31);
            x[q] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (s < S && f[q] > 0.f) {
              uint32_t ra;
              asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(own), "r"(s));
              x[q] = ld_cluster_f4(ra);
            }
          }
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            acc.x += f[q] * x[q].x;
            acc.y += f[q] * x[q].y;
            acc.z += f[q] * x[q].z;
            acc.w += f[q] * x[q].w;
          }
        }
        const size_t row = (size_t)blockIdx.z * p.Hq + (size_t)blockIdx.y * G + h;
        const float inv = (Wl > 0.f) ? 1.f / Wl : 0.f;
        *reinterpret_cast<float4*>(p.out + row * kHeadDim + lane * 4) =
            make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
        if (lane == 0) {
          p.lse[row] = (Wl > 0.f) ? (M + log2f(Wl)) * 0.6931471805599453f : -INFINITY;
          if (p.blocks_consumed) p.blocks_consumed[row] = ts;
        }
      }
      __syncwarp();
      mbar_arrive_if(fin4_bar, lane == 0);
      if (warp == 0) {  // every read of the other CTAs' records is done: release them
        if (!mbar_wait_bounded(fin4_bar, 0, nullptr) && lane == 0) dev_error(p.status, SKV_DEV_TIMEOUT);
        __syncwarp();
        if (lane >= 1 && lane < S) cluster_arrive_remote(cluster_addr(release_bar, lane));
      }
    }
  } else if (warp == 0) {
    // stay resident (shared memory valid) until rank 0 has read this piece
    if (!mbar_wait_cluster(release_bar, 0, 8 * kWaitLimitNs) && lane == 0) dev_error(p.status, SKV_DEV_TIMEOUT);
  }
}

template <int G>
constexpr int nw_for() {
  return G == 8 ? 8 : SKV_CONSUMER_WARPS;
}
template <int G>
constexpr int minb_for() {
  return G == 8 ? 1 : SKV_CTAS_PER_SM;
}

template <int G>
int launch_t(const DecodeParams& p, cudaStream_t st) {
  constexpr int NW = nw_for<G>();
  constexpr int MINB = minb_for<G>();
  using C = Cfg<G, NW, MINB>;
  auto kern = decode_kernel<G, NW, MINB>;
  // Set the shared-memory attribute once per device (not inside a capture).
  static std::atomic<bool> attr_set[64];  // per device; racing first calls only repeat the set-up
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return (int)cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::TOTAL);
    if (err != cudaSuccess) return (int)err;
    attr_set[dev] = true;
  }
  if (p.sched == SCHED_PERSISTENT) {
    kern<<<dim3(p.n_ctas, 1, 1), C::THREADS, C::TOTAL, st>>>(p);
    return (int)cudaGetLastError();
  }
  // split schedule: one cluster of n_splits CTAs per group (<= 16; above 8
  // needs the non-portable size, allowed once per device).  The split count
  // only divides each group's walk (no workspace depends on it), so a cluster
  // shape that cannot be resident at once is halved until it can.
  if (p.n_splits < 1 || p.n_splits > kMaxClusterSplits) return (int)cudaErrorInvalidValue;
  static std::atomic<bool> np_set[64];
  if (!np_set[dev]) {
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (err != cudaSuccess) return (int)err;
    np_set[dev] = true;
  }
  DecodeParams q = p;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(C::THREADS, 1, 1);
  cfg.dynamicSmemBytes = C::TOTAL;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static std::atomic<int> fits[64][kMaxClusterSplits + 1];  // 1: resident at once, -1: not (per size)
  while (true) {
    cfg.gridDim = dim3(q.n_splits, q.Hkv, q.B);
    attr[0].val.clusterDim.x = q.n_splits;
    if (fits[dev][q.n_splits] == 0) {
      int n = 0;
      cudaError_t err = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
      if (err != cudaSuccess) return (int)err;
      fits[dev][q.n_splits] = n > 0 ? 1 : -1;
    }
    if (fits[dev][q.n_splits] > 0) break;
    if (q.n_splits == 1) return (int)cudaErrorInvalidConfiguration;
    q.n_splits = (q.n_splits + 1) / 2;
  }
  return (int)cudaLaunchKernelEx(&cfg, kern, q);
}

}  // namespace

int decode_consumer_warps(int G) {
  switch (G) {
    case 1: return nw_for<1>();
    case 2: return nw_for<2>();
    case 4: return nw_for<4>();
    default: return nw_for<8>();
  }
}

int decode_ctas_per_sm(int G) {
  switch (G) {
    case 1: return minb_for<1>();
    case 2: return minb_for<2>();
    case 4: return minb_for<4>();
    default: return minb_for<8>();
  }
}

int launch_decode(const DecodeParams& p, int G, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (G) {
    case 1: return launch_t<1>(p, st);
    case 2: return launch_t<2>(p, st);
    case 4: return launch_t<4>(p, st);
    case 8: return launch_t<8>(p, st);
    default: return (int)cudaErrorInvalidValue;
  }
}

// SM count of the current device (cached per device index; 148, a B200's,
// when no device can be queried, so that host-side planning works anywhere).
int num_sms() {
  static std::atomic<int> cached[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  int n = cached[dev].load();
  if (n == 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
    cached[dev].store(n);
  }
  return n;
}

}  // namespace skv
