// art.cu -- decode attention with run-time termination ("ART: Adaptive
// Run-time Termination" 2.2-2.4) for sm_100a.
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
//              kernel, and ends each chunk with a marker entry;
//   consumers  NW warps fold every block into their online-softmax states
//              (tile.cuh) and hand the judge, through a small ring of probe
//              slots, (m, l, O[0:8]) of their state after every block and
//              their whole state at the end of every chunk.  They never wait
//              for a decision;
//   judge      one warp combines the consumer warps' probes into the chunk-
//              local prefix after every block and the end-of-chunk states
//              into the chunk's record; then it waits for the previous
//              chunk's published prefix (m, l, O[0:8], run of passing tests,
//              blocks consumed or the stop) -- a decoupled look-back, as in
//              single-pass parallel prefix scans -- evaluates the test for all
//              CB blocks at once (lane t: block t; the patience run by warp
//              ballots) and publishes the inclusive prefix.
// The probe slots and the state area are a small per-CTA scratch in global
// memory (rewritten in place, so it stays in L2), which leaves the shared
// memory to a 3-stage ring at two CTAs per SM.
// A head that stops inside a chunk needs its state after the stop block, which
// the consumers have already passed: the judge posts a request, and at their
// next chunk boundary the consumers re-fold that chunk's blocks up to the stop
// for the stopping heads straight from the pool in global memory (once per
// head; the pages are usually still in L2); the judge overwrites the record.
// Chunks taken after every head of a group has stopped issue no loads.
// attn_decode's merge combines each head's records up to its stop chunk,
// which is exact.
#include "common.cuh"
#include "decode.cuh"
#include "tile.cuh"

// consumer warps per CTA, blocks per chunk, resident CTAs per SM (1 or 2)
#ifndef SKV_ART_WARPS
#define SKV_ART_WARPS 8
#endif
#ifndef SKV_ART_CHUNK
#define SKV_ART_CHUNK 16
#endif
#ifndef SKV_ART_CTAS_PER_SM
#define SKV_ART_CTAS_PER_SM 2
#endif

namespace skv {
namespace {

constexpr int kProbeFloats = 12;  // per (block, warp, head): m, l, pad, pad, O[0:8]
constexpr int kSlots = 8;         // probe ring depth (entries the consumers may run ahead)
constexpr int kReqs = 32;         // re-run requests in flight (at most one per chunk in the ring lag)
enum SlotKind : int { SLOT_TILE = 0, SLOT_END = 1, SLOT_FIX = 2, SLOT_QUIT = 3, SLOT_DONE = 4 };

constexpr size_t up16(size_t x) { return (x + 15) / 16 * 16; }

// Per-CTA scratch in global memory: probe slots [kSlots][NW][G][12] and the
// state area [NW][G][kRecFloats].
template <int G, int NW>
__host__ __device__ constexpr size_t scratch_floats() {
  return (size_t)kSlots * NW * G * kProbeFloats + (size_t)NW * G * kRecFloats;
}

template <int G, int NW, int CB, int ST>
struct ArtCfg {  // shared-memory layout
  using Ln = Lanes<G, NW>;
  static constexpr int RPW = Ln::RPW;
  static constexpr int THREADS = (NW + 2) * 32;  // consumers, producer, judge
  static constexpr size_t STAGE_BYTES = 2 * (size_t)kTileBytes;
  static constexpr int NBAR = 2 * ST + 1 + 2 * kSlots + 1;  // full, empty, fin, pfull, pfree, sfree
  static constexpr size_t OFF_BAR = ST * STAGE_BYTES;
  static constexpr size_t OFF_META = up16(OFF_BAR + NBAR * 8);        // int4 [ST]
  static constexpr size_t OFF_FLAGS = up16(OFF_META + ST * 16);       // int [4]
  static constexpr size_t OFF_TAG = OFF_FLAGS + 16;                   // int [kSlots][4]
  static constexpr size_t OFF_RTAG = OFF_TAG + kSlots * 16;           // int [kSlots]
  static constexpr size_t OFF_REQ = up16(OFF_RTAG + kSlots * 4);      // int [kReqs][4] + int [kReqs][G]
  static constexpr size_t OFF_P = up16(OFF_REQ + kReqs * 16 + (size_t)kReqs * G * 4);  // float2 [NW][RPW][G]
  static constexpr size_t OFF_A = OFF_P + (size_t)NW * RPW * G * 8;   // float2 [NW][G]
  static constexpr size_t OFF_LOCAL = up16(OFF_A + (size_t)NW * G * 8);  // float [CB][G][12]
  static constexpr size_t TOTAL = OFF_LOCAL + (size_t)CB * G * kProbeFloats * 4;
  static_assert(OFF_BAR % 16 == 0 && OFF_META % 16 == 0 && OFF_P % 16 == 0, "alignment");
  static_assert(OFF_A % 16 == 0 && OFF_LOCAL % 16 == 0, "alignment");
  static_assert(OFF_TAG % 16 == 0 && OFF_REQ % 16 == 0, "alignment");
  static_assert((RPW * G * 8) % 16 == 0 || G == 1, "pbuf rows");
  static_assert(CB >= 1 && CB <= 32, "one judge lane per block of a chunk");
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
  uint64_t* pfull = fin_bar + 1;      // [kSlots], one arrival per consumer warp
  uint64_t* pfree = pfull + kSlots;   // [kSlots], the judge's arrival
  uint64_t* sfree = pfree + kSlots;   // the judge has read the state area
  int4* meta = reinterpret_cast<int4*>(smem + C::OFF_META);  // {rows | 0 = end of chunk, group, chunk, block in chunk | blocks}
  volatile int* flags = reinterpret_cast<volatile int*>(smem + C::OFF_FLAGS);
  // flags[1]: abort (a bounded wait expired); flags[2]: consumers finished
  // (entries consumed + 1)
  volatile int* tag = reinterpret_cast<volatile int*>(smem + C::OFF_TAG);  // [kSlots][4]: kind, group, chunk, a
  volatile int* rtag = reinterpret_cast<volatile int*>(smem + C::OFF_RTAG);  // requests posted, per slot
  volatile int* req = reinterpret_cast<volatile int*>(smem + C::OFF_REQ);  // [kReqs][4]: group, chunk, vmask, stopmask
  volatile int* req_t = reinterpret_cast<volatile int*>(smem + C::OFF_REQ + kReqs * 16);  // [kReqs][G]
  float* local = reinterpret_cast<float*>(smem + C::OFF_LOCAL);
  float* probe = p.art_scratch + (size_t)blockIdx.x * scratch_floats<G, NW>();
  float* state = probe + (size_t)kSlots * NW * G * kProbeFloats;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int groups = p.B * p.Hkv;
  const Ctl ctl(p, G);
  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], NW);
    }
    mbar_init(fin_bar, NW);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(&pfull[s], NW);
      mbar_init(&pfree[s], 1);
    }
    mbar_init(sfree, 1);
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
    if (lane != 0) return;
    const uint64_t pol = policy_evict_first();
    const size_t head_stride = (size_t)kBlock * kHeadDim;
    int e = 0, ps = 0, round = 0;
    bool ok = true;
    auto emit = [&](int n, int g, int c, int w, int page, int kvh) -> bool {
      if (round >= 1 && !mbar_wait_bounded(&empty[ps], (round - 1) & 1, &flags[1])) {
        fail();
        return false;
      }
      meta[ps] = make_int4(n, g, c, w);
      if (n > 0) {
        unsigned char* sK = smem + ps * C::STAGE_BYTES;
        const size_t src = ((size_t)page * p.Hkv + kvh) * head_stride;
        mbar_arrive_expect_tx(&full[ps], (uint32_t)n * kRowBytes * 2);
        bulk_load(sK, p.k_pool + src, (uint32_t)n * kRowBytes, &full[ps], pol);
        bulk_load(sK + kTileBytes, p.v_pool + src, (uint32_t)n * kRowBytes, &full[ps], pol);
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
    while (ok) {
      const long long w = atomicAdd(ctl.counter, 1);
      if (w >= items) break;
      const int c = (int)(w / groups), g = (int)(w % groups);
      const int b = g / p.Hkv, kvh = g % p.Hkv;
      int L = p.seq_lens[b];
      if (L < 0 || L > p.max_seq_len) {
        if (c == 0 && kvh == 0) dev_error(p.status, SKV_DEV_BAD_SEQLEN);
        L = 0;
      }
      const int nb = (L + kBlock - 1) / kBlock;
      const int N = art_positions(p, L);
      if (c * CB >= N) continue;
      const int sc = *reinterpret_cast<volatile int*>(ctl.stop_chunk + g);
      if (sc != 0 && c >= sc) continue;  // every head stopped in an earlier chunk
      const int* ord = (p.mode == TRAV_ORDER) ? p.order + (size_t)g * p.order_len : nullptr;
      const int* bt = p.block_table + (size_t)b * p.max_blocks;
      const int pos0 = c * CB, npos = min(CB, N - pos0);
      for (int i = 0; i < npos && ok; ++i) {
        const int blk = art_block(p, ord, nb, pos0 + i, p.status);
        if (blk < 0) continue;
        const int page = bt[blk];
        if (page < 0 || page >= p.num_pages) {
          dev_error(p.status, SKV_DEV_BAD_PAGE);
          continue;
        }
        ok = emit(min(kBlock, L - blk * kBlock), g, c, i, page, kvh);
      }
      if (ok) ok = emit(0, g, c, npos, 0, 0);  // end of chunk
    }
    if (ok) emit(-1, -1, 0, 0, 0, 0);
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

  // ------------------------------------------------------------------ judge
  if (warp == NW + 1) {
    int kj = 0;     // probe-ring entries consumed
    int n_req = 0;  // re-run requests posted
    int n_fix = 0;  // re-runs received back
    // combine the state area into the records of `heads` of chunk (g, c)
    auto reduce_states = [&](int g, int c, uint32_t heads) {
      const size_t item = (size_t)g * p.art_maxc + c;
      for (int h = 0; h < G; ++h) {
        if (!((heads >> h) & 1u)) continue;
        float2 ml[NW];
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < NW; ++w) {
          ml[w] = *reinterpret_cast<const float2*>(state + (w * G + h) * kRecFloats + 128);
          if (ml[w].y > 0.f) M = fmaxf(M, ml[w].x);
        }
        float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
        float Ls = 0.f;
        if (M != -INFINITY) {
#pragma unroll
          for (int w = 0; w < NW; ++w) {
            const float f = (ml[w].y > 0.f) ? exp2f(ml[w].x - M) : 0.f;
            const float4 x = *reinterpret_cast<const float4*>(state + (w * G + h) * kRecFloats + lane * 4);
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
      __syncwarp();
      mbar_arrive_if(sfree, lane == 0);
    };

    // Look-back and the stopping rule for chunk (g, c): publishes the chunk's
    // inclusive prefix; returns the heads that stop in the chunk, their stop
    // blocks in st_out (-1: none).
    auto evaluate = [&](int g, int c, uint32_t vmask, int* st_out) -> uint32_t {
      const size_t item = (size_t)g * p.art_maxc + c;
      const int b = g / p.Hkv;
      int L = p.seq_lens[b];
      if (L < 0 || L > p.max_seq_len) L = 0;
      const int nch = (art_positions(p, L) + CB - 1) / CB;
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
      // every head's previous record in one round trip: word k of the group at lane k % 32
      float pw0 = 0.f, pw1 = 0.f, pw2 = 0.f;
      if (c > 0) {
        const float* src = p.art_lb + (item - 1) * G * kProbeFloats;
        if (lane < G * kProbeFloats) pw0 = __ldcg(src + lane);
        if (lane + 32 < G * kProbeFloats) pw1 = __ldcg(src + lane + 32);
        if (lane + 64 < G * kProbeFloats) pw2 = __ldcg(src + lane + 64);
      }
      uint32_t stopmask = 0;
      bool all = true;
      for (int h = 0; h < G; ++h) {
        float Pv[kProbeFloats];
#pragma unroll
        for (int k = 0; k < kProbeFloats; ++k) {
          const int idx = h * kProbeFloats + k;
          const float v = __shfl_sync(0xffffffffu, idx < 32 ? pw0 : (idx < 64 ? pw1 : pw2), idx & 31);
          Pv[k] = (c > 0) ? v : (k == 0 ? -INFINITY : 0.f);
        }
        const int P_run = __float_as_int(Pv[10]), P_state = __float_as_int(Pv[11]);
        float out[kProbeFloats];
#pragma unroll
        for (int k = 0; k < kProbeFloats; ++k) out[k] = Pv[k];
        if (P_state >= 0) {
          // chunk-local prefix after block t (lane t), then the global prefix
          const int t = lane;
          const bool valid = t < CB && ((vmask >> t) & 1u);
          float M = -INFINITY, Ls = 0.f, X[8];
#pragma unroll
          for (int d = 0; d < 8; ++d) X[d] = 0.f;
          if (valid) {
            const float* q = local + ((size_t)t * G + h) * kProbeFloats;
            M = q[0];
            Ls = q[1];
            const float4 x0 = *reinterpret_cast<const float4*>(q + 4);
            const float4 x1 = *reinterpret_cast<const float4*>(q + 8);
            X[0] = x0.x; X[1] = x0.y; X[2] = x0.z; X[3] = x0.w;
            X[4] = x1.x; X[5] = x1.y; X[6] = x1.z; X[7] = x1.w;
          }
          const float Mg = fmaxf(Pv[0], M);
          const float fa = (Pv[0] == -INFINITY) ? 0.f : exp2f(Pv[0] - Mg);
          const float fb = (M == -INFINITY) ? 0.f : exp2f(M - Mg);
          const float Lg = Pv[1] * fa + Ls * fb;
          const float invL = (Lg > 0.f) ? 1.f / Lg : 0.f;
          const float invP = (Pv[1] > 0.f) ? 1.f / Pv[1] : 0.f;
          float Xg[8], xn[8], xp[8];
#pragma unroll
          for (int d = 0; d < 8; ++d) {
            Xg[d] = Pv[2 + d] * fa + X[d] * fb;
            xn[d] = Xg[d] * invL;
          }
          // probe of the previous consumed block: the last valid lane below,
          // else the previous prefix
          const uint32_t below = vmask & ((1u << t) - 1u);
          const int pl = below ? 31 - __clz(below) : 0;
#pragma unroll
          for (int d = 0; d < 8; ++d) {
            const float v = __shfl_sync(0xffffffffu, xn[d], pl);
            xp[d] = below ? v : Pv[2 + d] * invP;
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
          const uint32_t passm = __ballot_sync(0xffffffffu, pass);
          const uint32_t failm = __ballot_sync(0xffffffffu, valid && !pass);
          const uint32_t upto = (2u << t) - 1u;  // lanes 0..t (wraps to all for t = 31)
          const uint32_t ff = failm & upto;
          int run;
          if (ff) {
            const int f = 31 - __clz(ff);
            run = __popc(passm & upto & ~((2u << f) - 1u));
          } else {
            run = P_run + __popc(passm & upto);
          }
          const uint32_t stopm = __ballot_sync(0xffffffffu, valid && run >= p.patience);
          const int total = P_state + __popc(vmask);
          if (stopm) {
            const int ts = __ffs(stopm) - 1;
            const int used = P_state + __popc(vmask & ((2u << ts) - 1u));
            out[10] = __int_as_float(0);
            out[11] = __int_as_float(-(used + 1));
            st_out[h] = ts;
            stopmask |= 1u << h;
            if (lane == 0) {
              ctl.consumed[(size_t)g * G + h] = used;
              ctl.head_stop[(size_t)g * G + h] = c + 1;
            }
          } else {
            all = false;
            const int last = vmask ? 31 - __clz(vmask) : -1;
            if (last >= 0) {
              out[0] = __shfl_sync(0xffffffffu, Mg, last);
              out[1] = __shfl_sync(0xffffffffu, Lg, last);
#pragma unroll
              for (int d = 0; d < 8; ++d) out[2 + d] = __shfl_sync(0xffffffffu, Xg[d], last);
              out[10] = __int_as_float(__shfl_sync(0xffffffffu, run, last));
            }
            out[11] = __int_as_float(total);
            if (lane == 0 && c == nch - 1) ctl.consumed[(size_t)g * G + h] = total;
          }
        }
        float* dst = p.art_lb + (item * G + h) * kProbeFloats;
        float mine = 0.f;
#pragma unroll
        for (int k = 0; k < kProbeFloats; ++k)
          if (lane == k) mine = out[k];
        if (lane < kProbeFloats) dst[lane] = mine;
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
      const int slot = kj % kSlots;
      if (!mbar_wait_bounded(&pfull[slot], (kj / kSlots) & 1, &flags[1])) {
        if (lane == 0) fail();
        break;
      }
      const int kind = tag[slot * 4], tg_g = tag[slot * 4 + 1], tg_c = tag[slot * 4 + 2],
                tg_a = tag[slot * 4 + 3];
      if (kind == SLOT_TILE) {
        // chunk-local prefix after block tg_a: combine the warps' states (lane: head, dim)
        const float* pr = probe + (size_t)slot * NW * G * kProbeFloats;
#pragma unroll
        for (int r = 0; r < (G * 8 + 31) / 32; ++r) {
          const int h = r * 4 + (lane >> 3), d = lane & 7;
          if (h < G) {
            float m[NW];
            float M = -INFINITY;
#pragma unroll
            for (int w = 0; w < NW; ++w) {
              m[w] = pr[(w * G + h) * kProbeFloats];
              M = fmaxf(M, m[w]);
            }
            float Ls = 0.f, X = 0.f;
            if (M != -INFINITY) {
#pragma unroll
              for (int w = 0; w < NW; ++w) {
                const float* q = pr + (w * G + h) * kProbeFloats;
                const float f = exp2f(m[w] - M);  // 0 for an empty warp state
                Ls += q[1] * f;
                X += q[4 + d] * f;
              }
            }
            float* dst = local + ((size_t)tg_a * G + h) * kProbeFloats;
            dst[4 + d] = X;
            if (d == 0) {
              dst[0] = M;
              dst[1] = Ls;
            }
          }
        }
      } else if (kind == SLOT_END) {
        reduce_states(tg_g, tg_c, (1u << G) - 1u);
        __syncwarp();  // every lane's local prefixes are visible
        int st[G];
        const uint32_t stopmask = evaluate(tg_g, tg_c, (uint32_t)tg_a, st);
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
            }
            ++n_req;
          }
        }
      } else if (kind == SLOT_FIX) {
        reduce_states(tg_g, tg_c, (uint32_t)tg_a);
        ++n_fix;
      }
      __syncwarp();
      if (lane == 0) rtag[slot] = n_req;
      __syncwarp();
      mbar_arrive_if(&pfree[slot], lane == 0);
      ++kj;
      if (kind == SLOT_DONE) break;
    }
    return;
  }

  // ------------------------------------------------------------------ consumers
  Warp<G, NW> W;
  W.setup(warp, lane);
  const int rb = warp * C::RPW;
  float2* pbuf = reinterpret_cast<float2*>(smem + C::OFF_P) + warp * C::RPW * G;
  float2* abuf = reinterpret_cast<float2*>(smem + C::OFF_A) + warp * G;
  int ks = 0;          // probe-ring entries posted
  int req_seen = 0;    // requests the judge had posted at the last slot handshake
  int req_done = 0;    // requests served
  int n_state = 0;     // uses of the state area
  bool ok = true;

  // Post one probe-ring entry; `fill(slot)` writes this warp's part first.
  // Every warp reads the judge's request count at the same handshake, so all
  // take the same decisions.
  auto post = [&](int kind, int g, int c, int a, auto&& fill) {
    const int slot = ks % kSlots;
    if (ks >= kSlots) {
      if (!mbar_wait_bounded(&pfree[slot], ((ks / kSlots) - 1) & 1, &flags[1])) {
        if (lane == 0) fail();
        ok = false;
      }
      req_seen = rtag[slot];
    }
    fill(slot);
    if (warp == 0 && lane == 0) {
      tag[slot * 4] = kind;
      tag[slot * 4 + 1] = g;
      tag[slot * 4 + 2] = c;
      tag[slot * 4 + 3] = a;
    }
    __syncwarp();
    mbar_arrive_if(&pfull[slot], lane == 0);
    ++ks;
  };
  auto no_fill = [](int) {};
  // this warp's whole state -> the state area (once the judge has read the last one)
  auto write_state = [&]() {
    if (n_state >= 1 && !mbar_wait_bounded(sfree, (n_state - 1) & 1, &flags[1])) {
      if (lane == 0) fail();
      ok = false;
    }
    ++n_state;
#pragma unroll
    for (int g2 = 0; g2 < G; ++g2) {
      float x0, x1, x2, x3;
      unpack2(W.acc[g2][0], x0, x1);
      unpack2(W.acc[g2][1], x2, x3);
      *reinterpret_cast<float4*>(state + (warp * G + g2) * kRecFloats + lane * 4) =
          make_float4(x0, x1, x2, x3);
    }
    if (W.owner) {
#pragma unroll
      for (int j = 0; j < Lanes<G, NW>::VPL; ++j)
        *reinterpret_cast<float2*>(state + (warp * G + W.hd[j]) * kRecFloats + 128) =
            make_float2(W.m_st[j], W.l_st[j]);
    }
  };

  // Re-fold of a chunk for the heads that stop in it (a request of the judge):
  // the chunk's blocks up to each head's stop block, from the pool.
  int rr = -1;  // request being served
  int rr_t = 0, rr_tmax = 0, rr_g = 0, rr_c = 0, rr_L = 0, rr_nb = 0, rr_kvh = 0;
  uint32_t rr_vm = 0, rr_stop = 0;
  const int* rr_ord = nullptr;
  const int* rr_bt = nullptr;
  int rr_st[G];
  uint32_t done_mask = 0;
  auto start_request = [&]() -> bool {
    if (req_done >= req_seen || !ok) return false;
    rr = req_done % kReqs;
    rr_g = req[rr * 4];
    rr_c = req[rr * 4 + 1];
    rr_vm = (uint32_t)req[rr * 4 + 2];
    rr_stop = (uint32_t)req[rr * 4 + 3];
    rr_tmax = -1;
#pragma unroll
    for (int h = 0; h < G; ++h) {
      rr_st[h] = req_t[rr * G + h];
      if ((rr_stop >> h) & 1u) rr_tmax = max(rr_tmax, rr_st[h]);
    }
    const int b = rr_g / p.Hkv;
    rr_kvh = rr_g % p.Hkv;
    rr_L = p.seq_lens[b];
    if (rr_L < 0 || rr_L > p.max_seq_len) rr_L = 0;
    rr_nb = (rr_L + kBlock - 1) / kBlock;
    rr_ord = (p.mode == TRAV_ORDER) ? p.order + (size_t)rr_g * p.order_len : nullptr;
    rr_bt = p.block_table + (size_t)b * p.max_blocks;
    rr_t = 0;
    W.reset();
    W.load_q(p.q, (size_t)b * p.Hq + (size_t)rr_kvh * G, p.qscale, lane);
    done_mask = ~rr_stop;
    return true;
  };

  int e = 0, s = 0;
  uint32_t ph = 0;
  int cur_g = -1, cur_c = -1;
  uint32_t vmask = 0;
  bool draining = false;  // the producer's end entry has been seen
  while (ok) {
    const unsigned char* sK;
    const unsigned char* sV;
    int nv, pos = 0;
    const bool from_ring = rr < 0;
    if (!from_ring) {
      while (rr_t <= rr_tmax && !((rr_vm >> rr_t) & 1u)) ++rr_t;
      if (rr_t > rr_tmax) {  // request complete: its states go to the judge
        write_state();
        post(SLOT_FIX, rr_g, rr_c, (int)rr_stop, no_fill);
        ++req_done;
        rr = -1;
        cur_g = -1;  // the registers were used: reload at the next block
        if (!start_request() && draining) {
          post(SLOT_DONE, 0, 0, 0, no_fill);
          break;
        }
        continue;
      }
      const int blk = art_block(p, rr_ord, rr_nb, rr_c * CB + rr_t, nullptr);
      const size_t off = ((size_t)rr_bt[blk] * p.Hkv + rr_kvh) * kBlock * kHeadDim;  // page validated at load
      sK = reinterpret_cast<const unsigned char*>(p.k_pool + off);
      sV = reinterpret_cast<const unsigned char*>(p.v_pool + off);
      nv = min(kBlock, rr_L - blk * kBlock) - rb;
    } else {
      if (!mbar_wait_bounded(&full[s], ph, &flags[1])) {
        if (lane == 0) fail();
        ok = false;
        break;
      }
      const int4 mt = meta[s];
      const int n = mt.x;
      if (n < 0) {
        // end of the traversal: once the judge has handled every chunk (the
        // QUIT entry's handshake), serve the last requests, then release it
        draining = true;
        post(SLOT_QUIT, 0, 0, 0, no_fill);
        const int slot = (ks - 1) % kSlots;
        if (!mbar_wait_bounded(&pfree[slot], ((ks - 1) / kSlots) & 1, &flags[1])) {
          if (lane == 0) fail();
          ok = false;
          break;
        }
        req_seen = rtag[slot];
        if (!start_request()) {
          post(SLOT_DONE, 0, 0, 0, no_fill);
          break;
        }
        continue;
      }
      if (mt.y != cur_g || mt.z != cur_c) {
        cur_g = mt.y;
        cur_c = mt.z;
        W.reset();
        const int b = cur_g / p.Hkv, kvh = cur_g % p.Hkv;
        W.load_q(p.q, (size_t)b * p.Hq + (size_t)kvh * G, p.qscale, lane);
        vmask = 0;
        done_mask = 0;
      }
      if (n == 0) {  // end of chunk
        mbar_arrive_if(&empty[s], lane == 0);
        ++e;
        if (++s == ST) {
          s = 0;
          ph ^= 1u;
        }
        write_state();
        post(SLOT_END, cur_g, cur_c, (int)vmask, no_fill);
        start_request();
        continue;
      }
      sK = smem + s * C::STAGE_BYTES;
      sV = sK + kTileBytes;
      nv = n - rb;
      pos = mt.w;
    }
    if (nv >= C::RPW) fold_tile<G, NW, false>(W, sK, sV, nv, done_mask, pbuf, abuf);
    else fold_tile<G, NW, true>(W, sK, sV, nv, done_mask, pbuf, abuf);
    if (from_ring) {
      mbar_arrive_if(&empty[s], lane == 0);
      ++e;
      if (++s == ST) {
        s = 0;
        ph ^= 1u;
      }
      // this warp's running state after block `pos` of the chunk
      vmask |= 1u << pos;
      post(SLOT_TILE, cur_g, cur_c, pos, [&](int slot) {
        float* pw = probe + ((size_t)slot * NW + warp) * G * kProbeFloats;
        if (W.owner) {
#pragma unroll
          for (int j = 0; j < Lanes<G, NW>::VPL; ++j)
            *reinterpret_cast<float2*>(pw + W.hd[j] * kProbeFloats) = make_float2(W.m_st[j], W.l_st[j]);
        }
        if (lane < 2) {
#pragma unroll
          for (int g2 = 0; g2 < G; ++g2) {
            float x0, x1, x2, x3;
            unpack2(W.acc[g2][0], x0, x1);
            unpack2(W.acc[g2][1], x2, x3);
            *reinterpret_cast<float4*>(pw + g2 * kProbeFloats + 4 + lane * 4) = make_float4(x0, x1, x2, x3);
          }
        }
      });
    } else {
#pragma unroll
      for (int h = 0; h < G; ++h)
        if (rr_st[h] == rr_t) done_mask |= 1u << h;
      ++rr_t;
    }
  }
  __syncwarp();
  mbar_arrive_if(fin_bar, lane == 0);
  if (warp == 0) {
    if (!mbar_wait_bounded(fin_bar, 0, nullptr) && lane == 0) dev_error(p.status, SKV_DEV_TIMEOUT);
    if (lane == 0) flags[2] = (flags[1] != 0) ? 1 : e + 1;
  }
}

// Chunk length, resident CTAs per SM, and the deepest ring (up to 6 stages)
// that fits in the shared memory of one CTA.
template <int G> constexpr int art_cb() { return SKV_ART_CHUNK; }
template <int G> constexpr int art_minb() { return G == 8 ? 1 : SKV_ART_CTAS_PER_SM; }
template <int G, int NW>
constexpr int art_st() {
  const size_t budget = (art_minb<G>() == 2 ? 113 : 227) * 1024;
  int st = 6;
  while (st > 2 && ArtCfg<G, NW, art_cb<G>(), 6>::TOTAL - (size_t)(6 - st) * 2 * kTileBytes > budget)
    --st;
  return st;
}

template <int G>
int launch_art_t(const DecodeParams& p, cudaStream_t st) {
  constexpr int NW = SKV_ART_WARPS, CB = art_cb<G>(), ST = art_st<G, NW>(), MINB = art_minb<G>();
  using C = ArtCfg<G, NW, CB, ST>;
  static_assert(C::TOTAL <= (MINB == 2 ? 113 : 227) * 1024, "shared memory budget");
  auto kern = art_kernel<G, NW, CB, ST, MINB>;
  static bool attr_set[64] = {};
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

}  // namespace

int art_ctas_per_sm(int G) { return G == 8 ? art_minb<8>() : art_minb<4>(); }

int art_chunk_blocks(int G) {
  switch (G) {
    case 1: return art_cb<1>();
    case 2: return art_cb<2>();
    case 4: return art_cb<4>();
    default: return art_cb<8>();
  }
}

size_t art_scratch_bytes_per_cta(int G) {
  constexpr int NW = SKV_ART_WARPS;
  switch (G) {
    case 1: return scratch_floats<1, NW>() * 4;
    case 2: return scratch_floats<2, NW>() * 4;
    case 4: return scratch_floats<4, NW>() * 4;
    default: return scratch_floats<8, NW>() * 4;
  }
}

int launch_art(const DecodeParams& p, int G, void* stream) {
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  switch (G) {
    case 1: return launch_art_t<1>(p, st);
    case 2: return launch_art_t<2>(p, st);
    case 4: return launch_art_t<4>(p, st);
    case 8: return launch_art_t<8>(p, st);
    default: return (int)cudaErrorInvalidValue;
  }
}

}  // namespace skv
