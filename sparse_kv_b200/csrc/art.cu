// art.cu -- decode attention with run-time termination ("ART (Attention
// Run-time Termination)" 2.2-2.4) for sm_100a.
//
// Traversal of a KV group: position 0 is block 0 (the attention sink, always
// consumed), then the caller's block list without block 0, or every other
// block most recent first.  After each block the probe x_t = (O / l)[0:8] of
// every query head is compared with x_{t-1}; a head stops once both the
// relative norm change and 1 - cos stay below tau and phi for `patience`
// consecutive blocks, and its output is the attention over the blocks it
// consumed.
//
// The test is sequential along a head's traversal, but its inputs are not: the
// probe after block t is the online-softmax combination of every block up to
// t, and that combination is associative.  So the traversal is cut into chunks
// of CB blocks, and persistent CTAs take (chunk, group) items in chunk-major
// order from an atomic counter.  Three roles per CTA:
//   producer   one lane streams each chunk's blocks through a TMA ring
//              (bulk copies, no multicast), exactly like the plain decode
//              kernel; the chunk's last tile carries its end (a chunk that
//              loads nothing, or is cut short, ends with a marker entry).  The
//              next item is taken and its pages looked up while the current
//              chunk's first tiles are in flight;
//   consumers  NW warps fold every block into their online-softmax states
//              (tile.cuh) and leave (m, l, O[0:8]) of their state after every
//              block in a per-CTA scratch area; at the end of a chunk each
//              warp writes its whole state and posts the chunk to the arbiter.
//              They never meet and never wait for a decision;
//   arbiter    one warp combines the warps' probes into the chunk-local prefix
//              after every block (lane = (block, head)), waits for the
//              previous chunk's published prefix (m, l, O[0:8], run of passing
//              tests, blocks consumed or the stop) -- a decoupled look-back,
//              as in single-pass parallel prefix scans -- evaluates the test
//              for all CB blocks at once (lane t: block t; the patience run by
//              warp ballots) and publishes the inclusive prefix; only then does
//              it reduce the warps' states into the chunk's record, which no
//              decision needs.
// Posts rotate through kPosts buffers, so the consumers run up to kPosts - 1
// chunks ahead of the arbiter, which may wait on other CTAs' look-back.  The probes and states live in global memory rewritten in place
// (they stay in L2), which leaves the shared memory to a 3-stage ring at two
// CTAs per SM.
// A head that stops inside a chunk needs its state after the stop block, which
// the consumers have already passed: the arbiter queues a request, the producer
// streams that chunk's blocks up to the stop once more through the ring (the
// pages are usually still in L2) as tagged tiles, and the consumers fold them
// for the stopping heads only; the arbiter overwrites the record.
// Chunks taken after every head of a group has stopped issue no loads, and a
// chunk in flight is cut short (checked every 8 tiles).  An optional gate
// (DecodeParams::art_ahead) holds a group's chunk c until chunk c - ahead - 1
// is decided, bounding the reads past a stop at the price of idle CTAs.
// attn_decode's merge combines each head's records up to its stop chunk,
// which is exact.
#include "common.cuh"
#include "decode.cuh"
#include "tile.cuh"

// consumer warps per CTA, resident CTAs per SM (1 or 2); SKV_ART_CHUNK forces the chunk length
#ifndef SKV_ART_WARPS
#define SKV_ART_WARPS 8
#endif
#ifndef SKV_ART_CTAS_PER_SM
#define SKV_ART_CTAS_PER_SM 2
#endif
// post buffers between the consumers and the arbiter: the consumers run up to
// SKV_ART_POSTS - 1 chunks ahead of the arbiter's decisions
#ifndef SKV_ART_POSTS
#define SKV_ART_POSTS 3
#endif

namespace skv {
namespace {

constexpr int kProbeFloats = 12;  // per (block, warp, head): m, l, pad, pad, O[0:8]
constexpr int kReqs = 32;         // re-run requests in flight (a few chunks' worth)
enum PostKind : int { POST_END = 1, POST_FIX = 2, POST_QUIT = 3, POST_DONE = 4 };
// ring entry tags (meta.w): block in chunk (bits 0..7), request slot (8..15), first
// entry of an item, last chunk of the group, last tile of the chunk, re-fold flag
constexpr int kFirstTag = 1 << 27;
constexpr int kLastChunkTag = 1 << 28;
constexpr int kLastTag = 1 << 29;
constexpr int kFixTag = 1 << 30;
constexpr int kDrainEntry = -2;  // meta.x of the entry that ends the items (before re-folds)

constexpr size_t up16(size_t x) { return (x + 15) / 16 * 16; }
constexpr int kPosts = SKV_ART_POSTS;
static_assert(kPosts >= 2 && kPosts <= 8, "post buffers");

// Per-CTA scratch in global memory, one buffer per post: probes
// [kPosts][CB][NW][G][12] and states [kPosts][NW][G][kRecFloats].
template <int G, int NW, int CB>
__host__ __device__ constexpr size_t probe_floats() {
  return (size_t)CB * NW * G * kProbeFloats;
}
template <int G, int NW, int CB>
__host__ __device__ constexpr size_t scratch_floats() {
  return kPosts * probe_floats<G, NW, CB>() + kPosts * (size_t)NW * G * kRecFloats;
}

template <int G, int NW, int CB, int ST>
struct ArtCfg {  // shared-memory layout
  using Ln = Lanes<G, NW>;
  static constexpr int RPW = Ln::RPW;
  static constexpr int THREADS = (NW + 2) * 32;  // consumers, producer, arbiter
  // a stage: K rows, V rows, and the group's q rows (loaded with a chunk's first block)
  static constexpr size_t STAGE_BYTES = 2 * (size_t)kTileBytes + (size_t)G * kRowBytes;
  static constexpr int NBAR = 2 * ST + 1 + 2 * kPosts;  // full, empty, fin, posted[], freed[]
  static constexpr size_t OFF_BAR = ST * STAGE_BYTES;
  static constexpr size_t OFF_META = up16(OFF_BAR + NBAR * 8);        // int4 [ST]
  static constexpr size_t OFF_FLAGS = up16(OFF_META + ST * 16);       // int [4]
  static constexpr size_t OFF_TAG = OFF_FLAGS + 16;                   // int [kPosts][4]
  static constexpr size_t OFF_REQ = OFF_TAG + 16 * kPosts;            // int [kReqs][4] + int [kReqs][G]
  static constexpr size_t OFF_P = up16(OFF_REQ + kReqs * 16 + (size_t)kReqs * G * 4);  // float2 [NW][RPW][G]
  static constexpr size_t OFF_A = OFF_P + (size_t)NW * RPW * G * 8;   // float2 [NW][G]
  static constexpr size_t OFF_WCTL = up16(OFF_A + (size_t)NW * G * 8);  // int [NW][8]
  static constexpr size_t OFF_LOCAL = OFF_WCTL + (size_t)NW * 8 * 4;    // float [CB][G][12] (arbiter)
  static constexpr size_t TOTAL = OFF_LOCAL + (size_t)CB * G * kProbeFloats * 4;
  static_assert(OFF_BAR % 16 == 0 && OFF_META % 16 == 0 && OFF_P % 16 == 0, "alignment");
  static_assert(OFF_A % 16 == 0 && OFF_WCTL % 16 == 0 && OFF_LOCAL % 16 == 0, "alignment");
  static_assert(OFF_TAG % 16 == 0 && OFF_REQ % 16 == 0, "alignment");
  static_assert((RPW * G * 8) % 16 == 0 || G == 1, "pbuf rows");
  static_assert(CB >= 1 && CB <= 32, "one arbiter lane per block of a chunk");
  static_assert(G * kProbeFloats <= 96, "look-back records of a group in three loads per lane");
};

// Block at traversal position `pos` of a sequence with nb blocks; -1 for a
// position that holds no block (block 0 again, or an invalid entry).
__device__ __forceinline__ int art_block(const DecodeParams& p, const int* ord, int nb, int pos,
                                         uint32_t* status) {
  if (pos == 0) return 0;
  if (p.mode != TRAV_ORDER) return nb - pos;
  const int j = ord[pos - 1];
  if (j == 0) return -1;  // block 0 is always first; a later mention adds nothing
  if (j < 0 || j >= nb) {
    if (status) dev_error(status, SKV_DEV_BAD_ORDER);
    return -1;
  }
  return j;
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
  asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// ctl layout (zeroed before every launch): [0] item counter, [4 ..) stop
// chunk + 1 per group (0: running), ready flags [group][chunk], blocks
// consumed [group][G], stop chunk + 1 per head [group][G].
struct Ctl {
  int* counter;
  int* stop_chunk;
  int* ready;
  int* consumed;
  int* head_stop;
  __device__ Ctl(const DecodeParams& p, int G) {
    const int groups = p.B * p.Hkv;
    counter = p.art_ctl;
    stop_chunk = p.art_ctl + 4;
    ready = stop_chunk + groups;
    consumed = ready + (size_t)groups * p.art_maxc;
    head_stop = consumed + (size_t)groups * G;
  }
};

template <int G, int NW, int CB, int ST, int MINB>
__global__ void __launch_bounds__(ArtCfg<G, NW, CB, ST>::THREADS, MINB) art_kernel(const DecodeParams p) {
  using C = ArtCfg<G, NW, CB, ST>;
  extern __shared__ __align__(128) unsigned char smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + ST;
  uint64_t* fin_bar = empty + ST;
  uint64_t* posted = fin_bar + 1;   // [kPosts] a post is ready (one arrival per consumer warp)
  uint64_t* freed = posted + kPosts;  // [kPosts] the arbiter is done with a post
  int4* meta = reinterpret_cast<int4*>(smem + C::OFF_META);  // {rows | 0 = end of chunk, group, chunk, block in chunk | blocks}
  volatile int* flags = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  // flags[0]: re-fold requests posted by the arbiter; flags[1]: abort (a bounded
  // wait expired); flags[2]: consumers finished (entries consumed + 1);
  // flags[3]: the arbiter has handled every chunk (no more requests)
  volatile int* tag = reinterpret_cast<volatile int*>(smem + C::OFF_TAG);    // [kPosts][4]: kind, group, chunk, a
  volatile int* req = reinterpret_cast<volatile int*>(smem + C::OFF_REQ);  // [kReqs][4]: group, chunk, vmask, stopmask
  volatile int* req_t = reinterpret_cast<volatile int*>(smem + C::OFF_REQ + kReqs * 16);  // [kReqs][G]
  float* probe = p.art_scratch + (size_t)blockIdx.x * scratch_floats<G, NW, CB>();  // [kPosts][CB][NW][G][12]
  float* state = probe + kPosts * probe_floats<G, NW, CB>();                       // [kPosts][NW][G][132]
  float* local = reinterpret_cast<float*>(smem + C::OFF_LOCAL);                    // [CB][G][12]

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int groups = p.B * p.Hkv;
  const Ctl ctl(p, G);
  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NW);
    }
    mbar_init(fin_bar, NW);
    for (int i = 0; i < kPosts; ++i) {
      mbar_init(&posted[i], NW);
      mbar_init(&freed[i], 1);
    }
    flags[0] = flags[1] = flags[2] = flags[3] = 0;
    fence_barrier_init();
  }
  __syncthreads();
  auto fail = [&]() {
    if (flags[1] == 0) {
      dev_error(p.status, SKV_DEV_TIMEOUT);
      flags[1] = 1;
    }
  };

  // ------------------------------------------------------------------ producer
  if (warp == NW) {
    // The whole warp looks up a chunk's pages (lane i: block i); lane 0 issues
    // the copies.  The next item is taken one ahead, so the atomic's latency
    // overlaps the current chunk.
    const uint64_t pol = policy_evict_first();
    const size_t head_stride = (size_t)kBlock * kHeadDim;
    int e = 0, ps = 0, round = 0;
    bool ok = true;
    auto emit = [&](int n, int g, int c, int w, int page, int kvh, const uint16_t* qsrc) -> bool {
      if (round >= 1 && !mbar_wait_bounded(&empty[ps], (round - 1) & 1, &flags[1])) {
        fail();
        return false;
      }
      meta[ps] = make_int4(n, g, c, w);
      if (n > 0) {
        unsigned char* sK = smem + ps * C::STAGE_BYTES;
        const size_t src = ((size_t)page * p.Hkv + kvh) * head_stride;
        const uint32_t qbytes = qsrc ? (uint32_t)G * kRowBytes : 0u;
        mbar_arrive_expect_tx(&full[ps], (uint32_t)n * kRowBytes * 2 + qbytes);
        bulk_load(sK, p.k_pool + src, (uint32_t)n * kRowBytes, &full[ps], pol);
        bulk_load(sK + kTileBytes, p.v_pool + src, (uint32_t)n * kRowBytes, &full[ps], pol);
        if (qsrc) bulk_load(sK + 2 * kTileBytes, qsrc, qbytes, &full[ps], pol);
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
    const long long items = (long long)groups * p.art_maxc;
    // Re-fold request r: the chunk's blocks up to the last stop block, tagged,
    // then a tagged end marker.  The request slot stays valid until the arbiter has
    // taken the re-fold's post (it never has more than kReqs outstanding).
    auto serve = [&](int r) {
      const int slot = r % kReqs;
      __threadfence_block();
      const int g = req[slot * 4], c = req[slot * 4 + 1];
      const uint32_t vm = (uint32_t)req[slot * 4 + 2], stop = (uint32_t)req[slot * 4 + 3];
      int tmax = -1;
      for (int h = 0; h < G; ++h)
        if ((stop >> h) & 1u) tmax = max(tmax, req_t[slot * G + h]);
      const int b = g / p.Hkv, kvh = g % p.Hkv;
      int L = p.seq_lens[b];
      if (L < 0 || L > p.max_seq_len) L = 0;
      const int nb = (L + kBlock - 1) / kBlock;
      const int* ord = (p.mode == TRAV_ORDER) ? p.order + (size_t)g * p.order_len : nullptr;
      const int* bt = p.block_table + (size_t)b * p.max_blocks;
      int n = 0, page = 0;
      if (lane <= tmax && ((vm >> lane) & 1u)) {
        const int blk = art_block(p, ord, nb, c * CB + lane, nullptr);
        page = bt[blk];  // validated when the block was first loaded
        n = min(kBlock, L - blk * kBlock);
      }
      const uint16_t* qsrc = p.q + ((size_t)b * p.Hq + (size_t)kvh * G) * kHeadDim;
      bool first = true;
      for (int t = 0; t <= tmax && ok; ++t) {
        if (!((vm >> t) & 1u)) continue;
        const int nt = __shfl_sync(0xffffffffu, n, t), pgt = __shfl_sync(0xffffffffu, page, t);
        int r1 = 1;
        if (lane == 0)
          r1 = emit(nt, g, c, kFixTag | (slot << 8) | t | (first ? kFirstTag : 0), pgt, kvh, first ? qsrc : nullptr);
        ok = __shfl_sync(0xffffffffu, r1, 0) != 0;
        first = false;
      }
      if (ok) {
        int r1 = 1;
        if (lane == 0) r1 = emit(0, g, c, kFixTag | (slot << 8) | (first ? kFirstTag : 0), 0, 0, nullptr);
        ok = __shfl_sync(0xffffffffu, r1, 0) != 0;
      }
    };
    int taken = 0;  // requests served
    auto serve_pending = [&]() {
      int posted = (lane == 0) ? flags[0] : 0;
      posted = __shfl_sync(0xffffffffu, posted, 0);
      while (ok && taken < posted) serve(taken++);
    };
    // An item looked up ahead of its emission (lane i: block i of the chunk).
    struct Item {
      long long w;
      int c, g, kvh, npos, n, page, lastc;
      uint32_t vm;
      bool skip;
    };
    auto resolve = [&](long long wi) -> Item {
      Item it;
      it.w = wi;
      it.c = it.g = it.kvh = it.npos = it.n = it.page = it.lastc = 0;
      it.vm = 0;
      it.skip = true;
      if (wi >= items) return it;
      it.c = (int)(wi / groups);
      it.g = (int)(wi % groups);
      const int b = it.g / p.Hkv;
      it.kvh = it.g % p.Hkv;
      int L = p.seq_lens[b];
      if (L < 0 || L > p.max_seq_len) {
        if (it.c == 0 && it.kvh == 0 && lane == 0) dev_error(p.status, SKV_DEV_BAD_SEQLEN);
        L = 0;
      }
      const int nb = (L + kBlock - 1) / kBlock;
      const int N = art_positions(p, L);
      if (it.c * CB >= N) return it;
      const int sc = *reinterpret_cast<volatile int*>(ctl.stop_chunk + it.g);
      if (__shfl_sync(0xffffffffu, sc != 0 && it.c >= sc, 0)) return it;  // every head stopped earlier
      it.skip = false;
      const int* ord = (p.mode == TRAV_ORDER) ? p.order + (size_t)it.g * p.order_len : nullptr;
      const int* bt = p.block_table + (size_t)b * p.max_blocks;
      const int pos0 = it.c * CB;
      it.npos = min(CB, N - pos0);
      it.lastc = pos0 + CB >= N ? kLastChunkTag : 0;
      int blk = -1;
      if (lane < it.npos) {
        blk = art_block(p, ord, nb, pos0 + lane, p.status);
        if (blk >= 0) {
          it.page = bt[blk];
          if (it.page < 0 || it.page >= p.num_pages) {
            dev_error(p.status, SKV_DEV_BAD_PAGE);
            blk = -1;
          } else {
            it.n = min(kBlock, L - blk * kBlock);
          }
        }
      }
      it.vm = __ballot_sync(0xffffffffu, blk >= 0);
      return it;
    };
    // 1: the group stopped at or before chunk c
    auto stopped_at = [&](int g, int c) -> bool {
      int s = 0;
      if (lane == 0) {
        const int sc = *reinterpret_cast<volatile int*>(ctl.stop_chunk + g);
        s = sc != 0 && c >= sc;
      }
      return __shfl_sync(0xffffffffu, s, 0) != 0;
    };
    long long w = (lane == 0) ? (long long)atomicAdd(ctl.counter, 1) : 0;
    Item cur = resolve(__shfl_sync(0xffffffffu, w, 0));
    while (ok) {
      serve_pending();
      if (cur.w >= items) break;
      // the next item is taken now and looked up while this chunk's first
      // tiles are in the ring, so the ring does not drain between chunks
      const long long w_next = (lane == 0) ? (long long)atomicAdd(ctl.counter, 1) : 0;
      bool have_next = false;
      Item nxt;
      auto prefetch = [&]() {
        if (!have_next) nxt = resolve(__shfl_sync(0xffffffffu, w_next, 0));
        have_next = true;
      };
      if (!cur.skip && cur.c > p.art_ahead) {
        // Speculation gate: start the chunk only once chunk c - ahead - 1 of the
        // group has been decided.  The awaited chunk has a smaller item number,
        // so the wait always ends.
        const int* rdy = ctl.ready + (size_t)cur.g * p.art_maxc + (cur.c - p.art_ahead - 1);
        const uint64_t t0 = globaltimer();
        while (true) {
          int st = 0;  // 0: wait, 1: go, 2: the group stopped, 3: abort
          if (lane == 0) {
            if (*reinterpret_cast<const volatile int*>(rdy) != 0) {
              st = 1;
            } else {
              const int sc = *reinterpret_cast<const volatile int*>(ctl.stop_chunk + cur.g);
              if (sc != 0 && cur.c >= sc) st = 2;
              else if (flags[1] != 0 || globaltimer() - t0 > kWaitLimitNs) st = 3;
            }
          }
          st = __shfl_sync(0xffffffffu, st, 0);
          if (st == 1) break;
          if (st == 2) {
            cur.skip = true;
            break;
          }
          if (st == 3) {
            if (lane == 0) fail();
            ok = false;
            break;
          }
          serve_pending();
          __nanosleep(128);
        }
        if (!ok) break;
      }
      if (!cur.skip && stopped_at(cur.g, cur.c)) cur.skip = true;  // stopped since the look-up
      if (!cur.skip) {
        const int b = cur.g / p.Hkv;
        const uint16_t* qsrc = p.q + ((size_t)b * p.Hq + (size_t)cur.kvh * G) * kHeadDim;
        const int last = cur.vm ? 31 - __clz(cur.vm) : -1;
        bool cut = false, any = false;  // (any: an entry of the item was issued)
        int sc_ahead = 0;  // lane 0: the group's stop chunk, loaded a tile before it is checked
        for (int i = 0; i < cur.npos && ok; ++i) {
          if (!((cur.vm >> i) & 1u)) continue;
          if ((i & 7) == 7 &&
              __shfl_sync(0xffffffffu, sc_ahead != 0 && cur.c >= sc_ahead, 0)) {  // cut the chunk short
            cut = true;
            break;
          }
          if ((i & 7) == 6 && lane == 0) sc_ahead = *reinterpret_cast<volatile int*>(ctl.stop_chunk + cur.g);
          const int ni = __shfl_sync(0xffffffffu, cur.n, i), pgi = __shfl_sync(0xffffffffu, cur.page, i);
          int r = 1;
          if (lane == 0)
            r = emit(ni, cur.g, cur.c, i | (i == last ? kLastTag | cur.lastc : 0) | (any ? 0 : kFirstTag),
                     pgi, cur.kvh, any ? nullptr : qsrc);
          any = true;
          ok = __shfl_sync(0xffffffffu, r, 0) != 0;
          prefetch();
        }
        if (ok && (cut || last < 0)) {  // no tile carried the end of the chunk
          int r = 1;
          // (the item's first entry when no tile was issued)
          if (lane == 0) r = emit(0, cur.g, cur.c, cur.npos | cur.lastc | (any ? 0 : kFirstTag), 0, 0, nullptr);
          ok = __shfl_sync(0xffffffffu, r, 0) != 0;
        }
      }
      prefetch();
      cur = nxt;
    }
    // no more items: the consumers hand the arbiter a QUIT post; once the arbiter has
    // handled every chunk, serve the last requests, then end the ring
    if (ok) {
      int r = 1;
      if (lane == 0) r = emit(kDrainEntry, -1, 0, 0, 0, 0, nullptr);
      ok = __shfl_sync(0xffffffffu, r, 0) != 0;
    }
    if (ok) {
      int done = 1;
      if (lane == 0) {
        const uint64_t t0 = globaltimer();
        while (flags[3] == 0) {
          if (flags[1] != 0 || globaltimer() - t0 > kWaitLimitNs) {
            fail();
            done = 0;
            break;
          }
        }
      }
      ok = __shfl_sync(0xffffffffu, done, 0) != 0;
    }
    if (ok) serve_pending();
    if (lane != 0) return;
    if (ok) emit(-1, -1, 0, 0, 0, 0, nullptr);
    // Copies the consumers never waited for (abort) must land before the CTA
    // exits: learn how many entries they consumed, then drain the rest.
    const uint64_t t_start = globaltimer();
    while (flags[2] == 0 && globaltimer() - t_start < kWaitLimitNs) {
    }
    int consumed = flags[2] - 1;
    if (consumed < 0 || flags[1] != 0) consumed = 0;
    for (int kk = (e - ST > consumed ? e - ST : consumed); kk < e; ++kk)
      mbar_wait_bounded(&full[kk % ST], (kk / ST) & 1, nullptr);
    return;
  }

  // ------------------------------------------------------------------ arbiter
  if (warp == NW + 1) {
    int kj = 0;     // posts consumed
    int n_req = 0;  // re-run requests posted
    int n_fix = 0;  // re-runs received back
    // Chunk-local prefix after every block of the chunk: combine the consumer
    // warps' running states.  Lane = one (block, head) pair; every load of a
    // half of the warps is issued at once (one L2 round trip per half).
    auto merge_probes = [&](const float* pr0, uint32_t vmask) {
      constexpr int NH = NW / 2;
      for (int i0 = 0; i0 < CB * G; i0 += 32) {
        const int i = i0 + lane, t = i / G, h = i % G;
        const bool valid = i < CB * G && ((vmask >> t) & 1u);
        float M = -INFINITY, Ls = 0.f, X[8];
#pragma unroll
        for (int d = 0; d < 8; ++d) X[d] = 0.f;
        if (valid) {
          const float* pr = pr0 + ((size_t)t * NW * G + h) * kProbeFloats;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            float2 ml[NH];
            float4 xa[NH], xb[NH];
#pragma unroll
            for (int w = 0; w < NH; ++w) {
              const float* q = pr + (size_t)(half * NH + w) * G * kProbeFloats;
              ml[w] = *reinterpret_cast<const float2*>(q);
              xa[w] = *reinterpret_cast<const float4*>(q + 4);
              xb[w] = *reinterpret_cast<const float4*>(q + 8);
            }
            float Mh = M;
#pragma unroll
            for (int w = 0; w < NH; ++w) Mh = fmaxf(Mh, ml[w].x);
            if (Mh != -INFINITY) {
              const float fo = exp2f(M - Mh);  // rescale what the first half gave (0 if none)
              Ls *= fo;
#pragma unroll
              for (int d = 0; d < 8; ++d) X[d] *= fo;
#pragma unroll
              for (int w = 0; w < NH; ++w) {
                const float f = exp2f(ml[w].x - Mh);  // 0 for an empty warp state
                Ls += ml[w].y * f;
                X[0] += xa[w].x * f; X[1] += xa[w].y * f; X[2] += xa[w].z * f; X[3] += xa[w].w * f;
                X[4] += xb[w].x * f; X[5] += xb[w].y * f; X[6] += xb[w].z * f; X[7] += xb[w].w * f;
              }
              M = Mh;
            }
          }
          float* dst = local + ((size_t)t * G + h) * kProbeFloats;
          *reinterpret_cast<float4*>(dst) = make_float4(M, Ls, 0.f, 0.f);
          *reinterpret_cast<float4*>(dst + 4) = make_float4(X[0], X[1], X[2], X[3]);
          *reinterpret_cast<float4*>(dst + 8) = make_float4(X[4], X[5], X[6], X[7]);
        }
      }
    };

    // combine the state area into the records of `heads` of chunk (g, c)
    auto reduce_states = [&](const float* st_area, int g, int c, uint32_t heads) {
      const size_t item = (size_t)g * p.art_maxc + c;
      for (int h = 0; h < G; ++h) {
        if (!((heads >> h) & 1u)) continue;
        // every load up front: one round trip to L2
        float2 ml[NW];
        float4 xs[NW];
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          ml[w] = *reinterpret_cast<const float2*>(st_area + (w * G + h) * kRecFloats + 128);
          xs[w] = *reinterpret_cast<const float4*>(st_area + (w * G + h) * kRecFloats + lane * 4);
        }
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w)
          if (ml[w].y > 0.f) M = fmaxf(M, ml[w].x);
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        float Ls = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < NW; ++w) {
            const float f = (ml[w].y > 0.f) ? exp2f(ml[w].x - M) : 0.f;
            const float4 x = xs[w];
            Ls += ml[w].y * f;
            o.x += x.x * f;
            o.y += x.y * f;
            o.z += x.z * f;
            o.w += x.w * f;
          }
        }
        float* rec = p.ws_rec + (item * G + h) * kRecFloats;
        *reinterpret_cast<float4*>(rec + lane * 4) = o;
        if (lane == 0) *reinterpret_cast<float4*>(rec + 128) = make_float4(M, Ls, 0.f, 0.f);
      }
    };

    // Look-back and the stopping rule for chunk (g, c): publishes the chunk's
    // inclusive prefix; returns the heads that stop in the chunk, their stop
    // blocks in st_out (-1: none).  SEG lanes per head (lane t: block t), so
    // 32 / SEG heads per pass.
    auto evaluate = [&](const float* loc, int g, int c, uint32_t vmask, bool last_chunk,
                        int* st_out) -> uint32_t {
      constexpr int SEG = CB <= 8 ? 8 : (CB <= 16 ? 16 : 32);
      constexpr int HPP = 32 / SEG;
      const size_t item = (size_t)g * p.art_maxc + c;
#pragma unroll
      for (int h = 0; h < G; ++h) st_out[h] = -1;
      // (1) the previous chunk's prefix: ready, or the group already stopped
      int lb = 1;
      if (c > 0 && lane == 0) {
        const uint64_t t0 = globaltimer();
        while (true) {
          if (ld_acquire(ctl.ready + item - 1) != 0) break;
          const int sc = *reinterpret_cast<volatile int*>(ctl.stop_chunk + g);
          if (sc != 0 && c >= sc) {
            lb = 2;
            break;
          }
          if (flags[1] != 0 || globaltimer() - t0 > kWaitLimitNs) {
            fail();
            lb = 2;
            break;
          }
        }
      }
      lb = __shfl_sync(0xffffffffu, lb, 0);
      if (lb == 2) return 0;  // nothing to publish: the group stopped before this chunk
      const int sub = lane / SEG, t = lane % SEG, base = sub * SEG;
      const uint32_t segmask = (SEG == 32) ? 0xffffffffu : ((1u << SEG) - 1u);
      uint32_t stopmask = 0;
      bool all = true;
      for (int h0 = 0; h0 < G; h0 += HPP) {
        const int h = h0 + sub;
        const bool hv = h < G;
        // previous inclusive prefix of head h: m, l, x[8], run, blocks or -(used + 1)
        float4 P0 = make_float4(-INFINITY, 0.f, 0.f, 0.f), P1 = make_float4(0.f, 0.f, 0.f, 0.f),
               P2 = make_float4(0.f, 0.f, 0.f, 0.f);
        if (c > 0 && hv) {
          const float4* src = reinterpret_cast<const float4*>(p.art_lb + ((item - 1) * G + h) * kProbeFloats);
          P0 = __ldcg(src);
          P1 = __ldcg(src + 1);
          P2 = __ldcg(src + 2);
        }
        const float Pm = P0.x, Pl = P0.y;
        const float Px[8] = {P0.z, P0.w, P1.x, P1.y, P1.z, P1.w, P2.x, P2.y};
        const int P_run = __float_as_int(P2.z), P_state = __float_as_int(P2.w);
        const bool live = hv && P_state >= 0;
        // chunk-local prefix after block t, then the global prefix
        const bool valid = live && t < CB && ((vmask >> t) & 1u);
        float M = -INFINITY, Ls = 0.f, X[8];
#pragma unroll
        for (int d = 0; d < 8; ++d) X[d] = 0.f;
        if (valid) {
          const float* q = loc + ((size_t)t * G + h) * kProbeFloats;
          const float2 ml = *reinterpret_cast<const float2*>(q);
          const float4 x0 = *reinterpret_cast<const float4*>(q + 4);
          const float4 x1 = *reinterpret_cast<const float4*>(q + 8);
          M = ml.x;
          Ls = ml.y;
          X[0] = x0.x; X[1] = x0.y; X[2] = x0.z; X[3] = x0.w;
          X[4] = x1.x; X[5] = x1.y; X[6] = x1.z; X[7] = x1.w;
        }
        const float Mg = fmaxf(Pm, M);
        const float fa = (Pm == -INFINITY) ? 0.f : exp2f(Pm - Mg);
        const float fb = (M == -INFINITY) ? 0.f : exp2f(M - Mg);
        const float Lg = Pl * fa + Ls * fb;
        const float invL = (Lg > 0.f) ? 1.f / Lg : 0.f;
        const float invP = (Pl > 0.f) ? 1.f / Pl : 0.f;
        float Xg[8], xn[8], xp[8];
#pragma unroll
        for (int d = 0; d < 8; ++d) {
          Xg[d] = Px[d] * fa + X[d] * fb;
          xn[d] = Xg[d] * invL;
        }
        // probe of the previous consumed block: the last valid lane below in
        // this head's segment, else the previous prefix
        const uint32_t below = vmask & ((1u << t) - 1u);
        const int pl = base + (below ? 31 - __clz(below) : 0);
#pragma unroll
        for (int d = 0; d < 8; ++d) {
          const float v = __shfl_sync(0xffffffffu, xn[d], pl);
          xp[d] = below ? v : Px[d] * invP;
        }
        const int gidx = P_state + __popc(below);  // consumed blocks before this one
        float nx = 0.f, np = 0.f, dd = 0.f;
#pragma unroll
        for (int d = 0; d < 8; ++d) {
          nx += xn[d] * xn[d];
          np += xp[d] * xp[d];
        }
        const float a = sqrtf(nx), bp = sqrtf(np);
        const float ia = (a > 0.f) ? 1.f / a : 0.f, ib = (bp > 0.f) ? 1.f / bp : 0.f;
#pragma unroll
        for (int d = 0; d < 8; ++d) {
          const float du = xn[d] * ia - xp[d] * ib;
          dd += du * du;
        }
        float d_s, d_c;
        if (bp == 0.f) d_s = (a == 0.f) ? 0.f : INFINITY;
        else d_s = fabsf(a - bp) * ib;
        if (a == 0.f || bp == 0.f) d_c = (a == 0.f && bp == 0.f) ? 0.f : 1.f;
        else d_c = 0.5f * dd;  // 1 - cos(x, x') = |x/|x| - x'/|x'||^2 / 2
        const bool pass = valid && gidx >= 1 && d_s < p.tau && d_c < p.phi;
        const uint32_t passm = (__ballot_sync(0xffffffffu, pass) >> base) & segmask;
        const uint32_t failm = (__ballot_sync(0xffffffffu, valid && !pass) >> base) & segmask;
        const uint32_t upto = (2u << t) - 1u;  // blocks 0..t (wraps to all for t = 31)
        const uint32_t ff = failm & upto;
        int run;
        if (ff) {
          const int f = 31 - __clz(ff);
          run = __popc(passm & upto & ~((2u << f) - 1u));
        } else {
          run = P_run + __popc(passm & upto);
        }
        const uint32_t stopm = (__ballot_sync(0xffffffffu, valid && run >= p.patience) >> base) & segmask;
        const int total = P_state + __popc(vmask);
        // the record of this chunk, written by one lane of the segment
        const int ts = stopm ? __ffs(stopm) - 1 : -1;
        const int last = vmask ? 31 - __clz(vmask) : -1;
        float4 R0 = P0, R1 = P1, R2 = P2;  // a head stopped earlier passes its record on
        int wl = 0;
        if (live) {
          if (ts >= 0) {
            const int used = P_state + __popc(vmask & ((2u << ts) - 1u));
            R2.z = __int_as_float(0);
            R2.w = __int_as_float(-(used + 1));
            wl = ts;
            if (t == ts) {
              ctl.consumed[(size_t)g * G + h] = used;
              ctl.head_stop[(size_t)g * G + h] = c + 1;
            }
          } else {
            if (last >= 0) {
              wl = last;
              R0 = make_float4(Mg, Lg, Xg[0], Xg[1]);
              R1 = make_float4(Xg[2], Xg[3], Xg[4], Xg[5]);
              R2 = make_float4(Xg[6], Xg[7], __int_as_float(run), __int_as_float(total));
            } else {
              R2.w = __int_as_float(total);
            }
            if (t == wl && last_chunk) ctl.consumed[(size_t)g * G + h] = total;
          }
        }
        if (hv && t == wl) {
          float4* dst = reinterpret_cast<float4*>(p.art_lb + (item * G + h) * kProbeFloats);
          dst[0] = R0;
          dst[1] = R1;
          dst[2] = R2;
        }
        // per-head outcome to every lane
#pragma unroll
        for (int s2 = 0; s2 < HPP; ++s2) {
          const int hh = h0 + s2;
          const int ts_h = __shfl_sync(0xffffffffu, live ? ts : -2, s2 * SEG);  // -2: stopped before
          if (hh < G) {
            if (ts_h >= 0) {
              stopmask |= 1u << hh;
              st_out[hh] = ts_h;
            } else if (ts_h == -1) {
              all = false;
            }
          }
        }
      }
      __threadfence();
      __syncwarp();
      if (lane == 0) {
        if (all && stopmask) {
          *reinterpret_cast<volatile int*>(ctl.stop_chunk + g) = c + 1;
          __threadfence();
        }
        st_release(ctl.ready + item, 1);
      }
      return stopmask;
    };

    while (true) {
      const int par = kj % kPosts;
      if (!mbar_wait_bounded(&posted[par], (kj / kPosts) & 1, &flags[1])) {
        if (lane == 0) fail();
        break;
      }
      const int kind = tag[par * 4] & 0xFF, tg_g = tag[par * 4 + 1], tg_c = tag[par * 4 + 2],
                tg_a = tag[par * 4 + 3];
      const bool last_chunk = (tag[par * 4] >> 16) & 1;
      const float* st_area = state + (size_t)par * NW * G * kRecFloats;
      if (kind == POST_END) {
        merge_probes(probe + (size_t)par * probe_floats<G, NW, CB>(), (uint32_t)tg_a);
        __syncwarp();  // the chunk-local prefixes are visible to every lane
        int st[G];
        const uint32_t stopmask = evaluate(local, tg_g, tg_c, (uint32_t)tg_a, last_chunk, st);
        if (stopmask) {
          if (n_req - n_fix >= kReqs) {
            if (lane == 0) fail();  // cannot happen: the consumers serve requests every chunk
          } else {
            const int r = n_req % kReqs;
            if (lane == 0) {
              req[r * 4] = tg_g;
              req[r * 4 + 1] = tg_c;
              req[r * 4 + 2] = tg_a;
              req[r * 4 + 3] = (int)stopmask;
#pragma unroll
              for (int h = 0; h < G; ++h) req_t[r * G + h] = st[h];
              __threadfence_block();
              flags[0] = n_req + 1;  // the producer serves it between items
            }
            ++n_req;
          }
        }
        // the chunk's records (after the decision: they are not on its path)
        reduce_states(st_area, tg_g, tg_c, (1u << G) - 1u);
      } else if (kind == POST_FIX) {
        reduce_states(st_area, tg_g, tg_c, (uint32_t)tg_a);
        ++n_fix;
      } else if (kind == POST_QUIT) {
        __syncwarp();
        if (lane == 0) flags[3] = 1;  // every chunk handled: no more requests
      }
      __syncwarp();
      mbar_arrive_if(&freed[par], lane == 0);
      ++kj;
      if (kind == POST_DONE) break;
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  Warp<G, NW> W;
  W.setup(warp, lane);
  const int rb = warp * C::RPW;
  float2* pbuf = reinterpret_cast<float2*>(smem + C::OFF_P) + warp * C::RPW * G;
  float2* abuf = reinterpret_cast<float2*>(smem + C::OFF_A) + warp * G;
  // Warp-uniform counters used at chunk boundaries live in shared memory (one
  // block per warp): the fold loop is register-bound.
  enum { W_KP = 0 };
  volatile int* wc = reinterpret_cast<volatile int*>(smem + C::OFF_WCTL) + warp * 8;
  wc[W_KP] = 0;      // posts made
  int kpar = 0;  // buffer of the next post (it holds the current item)
  bool ok = true;

  // Take the buffers of the next post (the arbiter is done with the post kPosts back).
  auto acquire = [&]() {
    const int kp = wc[W_KP];
    if (kp >= kPosts && !mbar_wait_bounded(&freed[kp % kPosts], ((kp / kPosts) - 1) & 1, &flags[1])) {
      if (lane == 0) fail();
      ok = false;
    }
  };
  auto publish = [&](int kind, int g, int c, int a) {
    const int kp = wc[W_KP];
    const int par = kp % kPosts;
    if (warp == 0 && lane == 0) {
      tag[par * 4] = kind;
      tag[par * 4 + 1] = g;
      tag[par * 4 + 2] = c;
      tag[par * 4 + 3] = a;
    }
    __syncwarp();
    mbar_arrive_if(&posted[par], lane == 0);
    wc[W_KP] = kp + 1;
    kpar = (kp + 1) % kPosts;
  };
  // this warp's whole state -> the state area of the current post
  auto write_state = [&]() {
    float* st_area = state + (size_t)(wc[W_KP] % kPosts) * NW * G * kRecFloats;
#pragma unroll
    for (int g2 = 0; g2 < G; ++g2) {
      float x0, x1, x2, x3;
      unpack2(W.acc[g2][0], x0, x1);
      unpack2(W.acc[g2][1], x2, x3);
      *reinterpret_cast<float4*>(st_area + (warp * G + g2) * kRecFloats + lane * 4) =
          make_float4(x0, x1, x2, x3);
    }
    if (W.owner) {
#pragma unroll
      for (int j = 0; j < Lanes<G, NW>::VPL; ++j)
        *reinterpret_cast<float2*>(st_area + (warp * G + W.hd[j]) * kRecFloats + 128) =
            make_float2(W.m_st[j], W.l_st[j]);
    }
  };

  int s = 0, e = 0;  // ring stage, ring entries consumed
  uint32_t ph = 0;
  uint32_t vmask = 0, done_mask = 0;
  auto release = [&]() {
    mbar_arrive_if(&empty[s], lane == 0);
    ++e;
    if (++s == ST) {
      s = 0;
      ph ^= 1u;
    }
  };
  while (ok) {
    if (!mbar_wait_bounded(&full[s], ph, &flags[1])) {
      if (lane == 0) fail();
      ok = false;
      break;
    }
    const int4 mt = meta[s];
    const int n = mt.x;
    if (n == -1) break;
    if (n == kDrainEntry) {  // no more items: let the arbiter finish, re-folds may follow
      release();
      acquire();
      publish(POST_QUIT, 0, 0, 0);
      continue;
    }
    const bool fix = (mt.w & kFixTag) != 0;
    const int slot = fix ? ((mt.w >> 8) & 0xFF) : -1;
    if (mt.w & kFirstTag) {
      // a new item (a chunk, or the re-fold of one): take the next post's buffers
      acquire();
      W.reset();
      if (n > 0)  // an item's first block carries the group's q rows
        W.load_q(reinterpret_cast<const uint16_t*>(smem + s * C::STAGE_BYTES + 2 * kTileBytes), 0,
                 p.qscale, lane);
      vmask = 0;
      __threadfence_block();
      done_mask = fix ? ~(uint32_t)req[slot * 4 + 3] : 0u;  // a re-fold folds its stopping heads only
    }
    if (n == 0) {  // end of the item
      release();
      write_state();
      publish(fix ? POST_FIX : (POST_END | ((mt.w & kLastChunkTag) ? 1 << 16 : 0)), mt.y, mt.z,
              fix ? req[slot * 4 + 3] : (int)vmask);
      continue;
    }
    const unsigned char* sK = smem + s * C::STAGE_BYTES;
    const unsigned char* sV = sK + kTileBytes;
    const int nv = n - rb;
    if (!fix) {  // the common path: every head folds the tile (a constant mask)
      if (nv >= C::RPW) fold_tile<G, NW, false>(W, sK, sV, nv, 0u, pbuf, abuf);
      else fold_tile<G, NW, true>(W, sK, sV, nv, 0u, pbuf, abuf);
    } else {     // a re-fold: only the stopping heads fold
      fold_tile<G, NW, true>(W, sK, sV, nv, done_mask, pbuf, abuf);
    }
    release();
    const int pos = mt.w & 0xFF;
    if (!fix) {
      // this warp's running state after block `pos` of the chunk (32-bit offsets:
      // the probes of every post together are far below 2^31 floats; the
      // per-head offsets are constants)
      vmask |= 1u << pos;
      float* pw = probe + (uint32_t)(kpar * (int)probe_floats<G, NW, CB>() +
                                     (pos * NW + warp) * (G * kProbeFloats));
      if (W.owner) {
#pragma unroll
        for (int j = 0; j < Lanes<G, NW>::VPL; ++j)
          *reinterpret_cast<float2*>(pw + W.hd[j] * kProbeFloats) = make_float2(W.m_st[j], W.l_st[j]);
      }
      if (lane < 2) {
        float* px = pw + 4 + lane * 4;
#pragma unroll
        for (int g2 = 0; g2 < G; ++g2) {
          float x0, x1, x2, x3;
          unpack2(W.acc[g2][0], x0, x1);
          unpack2(W.acc[g2][1], x2, x3);
          *reinterpret_cast<float4*>(px + g2 * kProbeFloats) = make_float4(x0, x1, x2, x3);
        }
      }
      if (mt.w & kLastTag) {  // the chunk's last tile: post the chunk
        write_state();
        publish(POST_END | ((mt.w & kLastChunkTag) ? 1 << 16 : 0), mt.y, mt.z, (int)vmask);
      }
    } else {
      // a stopping head takes no block after its stop block
#pragma unroll
      for (int h = 0; h < G; ++h)
        if (req_t[slot * G + h] == pos) done_mask |= 1u << h;
    }
  }
  if (ok) {  // release the arbiter
    acquire();
    publish(POST_DONE, 0, 0, 0);
  }
  __syncwarp();
  mbar_arrive_if(fin_bar, lane == 0);
  if (warp == 0) {
    if (!mbar_wait_bounded(fin_bar, 0, nullptr) && lane == 0) dev_error(p.status, SKV_DEV_TIMEOUT);
    if (lane == 0) flags[2] = (flags[1] != 0) ? 1 : e + 1;
  }
}

// Resident CTAs per SM, and the deepest ring (up to 6 stages) that fits in
// the shared memory of one CTA.
template <int G> constexpr int art_minb() { return G == 8 ? 1 : SKV_ART_CTAS_PER_SM; }
template <int G, int NW, int CB>
constexpr int art_st() {
  const size_t budget = (art_minb<G>() == 2 ? 113 : 227) * 1024;
  int st = 6;
  while (st > 2 && ArtCfg<G, NW, CB, 6>::TOTAL - (size_t)(6 - st) * 2 * kTileBytes > budget) --st;
  return st;
}

template <int G, int CB>
int launch_art_t(const DecodeParams& p, cudaStream_t st) {
  constexpr int NW = SKV_ART_WARPS, ST = art_st<G, NW, CB>(), MINB = art_minb<G>();
  using C = ArtCfg<G, NW, CB, ST>;
  static_assert(C::TOTAL <= (MINB == 2 ? 113 : 227) * 1024, "shared memory budget");
  static_assert(ST >= 3, "a ring of at least three stages");
  auto kern = art_kernel<G, NW, CB, ST, MINB>;
  static std::atomic<bool> attr_set[64];  // per device; racing first calls only repeat the set-up
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return (int)cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t err =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)C::TOTAL);
    if (err != cudaSuccess) return (int)err;
    attr_set[dev] = true;
  }
  kern<<<p.n_ctas, C::THREADS, C::TOTAL, st>>>(p);
  return (int)cudaGetLastError();
}

template <int G>
int launch_art_g(const DecodeParams& p, cudaStream_t st) {
  return p.art_chunk == 16 ? launch_art_t<G, 16>(p, st) : launch_art_t<G, 32>(p, st);
}

}  // namespace

int art_ctas_per_sm(int G) { return G == 8 ? art_minb<8>() : art_minb<4>(); }

// Chunk length: 32 blocks, or 16 when the speculation window would be large.
// About n_ctas / groups chunks of a group are in flight when one of its stops
// is decided, and all of them are read in vain; keep that within 1/12 of the
// traversal.  Shorter chunks cost more deciding per block, so they are used
// only where the window needs them.
int art_chunk_blocks(int G, long long n_ctas, long long groups, long long positions) {
  (void)G;
#ifdef SKV_ART_CHUNK
  return SKV_ART_CHUNK;
#else
  const double in_flight = (double)n_ctas / (double)(groups > 0 ? groups : 1);
  return (in_flight * 32.0 <= (double)positions / 12.0) ? 32 : 16;
#endif
}

size_t art_scratch_bytes_per_cta(int G, int CB) {
  constexpr int NW = SKV_ART_WARPS;
  const bool s = CB == 16;
  switch (G) {
    case 1: return (s ? scratch_floats<1, NW, 16>() : scratch_floats<1, NW, 32>()) * 4;
    case 2: return (s ? scratch_floats<2, NW, 16>() : scratch_floats<2, NW, 32>()) * 4;
    case 4: return (s ? scratch_floats<4, NW, 16>() : scratch_floats<4, NW, 32>()) * 4;
    default: return (s ? scratch_floats<8, NW, 16>() : scratch_floats<8, NW, 32>()) * 4;
  }
}

int launch_art(const DecodeParams& p, int G, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (p.art_chunk != 16 && p.art_chunk != 32) return (int)cudaErrorInvalidValue;
  switch (G) {
    case 1: return launch_art_g<1>(p, st);
    case 2: return launch_art_g<2>(p, st);
    case 4: return launch_art_g<4>(p, st);
    case 8: return launch_art_g<8>(p, st);
    default: return (int)cudaErrorInvalidValue;
  }
}

}  // namespace skv
