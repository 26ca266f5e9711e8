// chunk.cu -- attention of a query chunk (q_tokens > 1) on the tcgen05 tensor
// cores of sm_100a.
//
// A KV group's G query heads and Tq chunk tokens form G*Tq rows (row r =
// token r / G, head r % G), a dense contraction against the keys.  One CTA
// computes 128 rows against one key range (a shard: "Pulsar Attention" Phase
// 2 local attention; or the chunk's own keys under a causal mask) and writes
// that partial's normalised O and log-sum-exp; partials combine exactly with
// attn_merge_lse.
//
// Warp roles (11 warps):
//   warps 0, 10 producers: TMA tensor loads (128B swizzle, no multicast) of the
//               K rows (warp 0) and V rows (warp 10) of 128-key tiles into two
//               separate 2-stage rings (a K stage frees after Q K^T, a V stage
//               after P V, so the next keys load while the softmax runs)
//   warp 1      MMA: allocates 512 TMEM columns, issues tcgen05.mma for
//               S = Q K^T into two ping-pong S buffers of 128 fp32 columns and,
//               per key half h, O_h += P_h V_h (two accumulators of 128 fp32
//               columns; the A operand P_h is read from TMEM, where the
//               softmax wrote it over the S columns it came from), and commits
//               to mbarriers
//   warps 2..9  softmax: two threads per row (TMEM lane), one per 64-key half
//               of every tile (warps 2..5 the low half, 6..9 the high half; a
//               warp may only touch its own quarter of the TMEM lanes, and both
//               warps of a pair sit on the same quarter).  Each thread runs its
//               own online softmax over its half's keys: reads its half of the
//               S row with tcgen05.ld, masks, keeps its running max, rescales
//               its accumulator O_h in TMEM only when the max grows by more than
//               2^8 (the scale is applied consistently to O_h and l_h, so the
//               result stays exact), and writes P_h with tcgen05.st as two bf16
//               terms (hi + lo, about 16 significant bits together), each over
//               32 of the half's 64 S columns.  The two halves meet once, at the
//               end, to combine (m, l, O) of the row exactly.
// Operands: Q and K K-major, V MN-major, in the canonical 128B-swizzle layout
// (8-row x 128-byte atoms, 1024-byte aligned) in shared memory; P in TMEM
// (row = lane, two bf16 keys per 32-bit column, hi and lo terms); bf16 x bf16
// -> fp32.
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"
#include "decode.cuh"

namespace skv {
namespace {

constexpr int BM = 128;                         // rows per CTA
constexpr int BN = 128;                         // keys per tile
constexpr int kChunkWarps = 11;
constexpr int kChunkThreads = kChunkWarps * 32;
constexpr int kHalf = BM * 64 * 2;              // one 64-column half of a 128-row tile: 16 KiB
constexpr int kTile = 2 * kHalf;                // 32 KiB
constexpr int kStages = 2;
constexpr uint32_t kTmemCols = 512;  // S0 [0,128), S1 [128,256), O_0 [256,384), O_1 [384,512)
constexpr uint32_t kColO = 256;       // O_h at kColO + h * 128

constexpr size_t OFF_Q = 0;
constexpr size_t OFF_K = OFF_Q + (size_t)kTile;      // K stage s at +s*kTile
constexpr size_t OFF_V = OFF_K + (size_t)kStages * kTile;  // V stage s at +s*kTile
constexpr size_t OFF_BAR = OFF_V + (size_t)kStages * kTile;
// k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], p_full[2], o_done[2],
// xbar[4] (one per softmax warp pair)
constexpr int NBAR = 18;
constexpr size_t OFF_XCH = OFF_BAR + NBAR * 8;       // float [2 parity][2 halves][128 rows]
constexpr size_t OFF_TMEM = OFF_XCH + 2 * 2 * BM * 4;
constexpr size_t OFF_FLAG = OFF_TMEM + 16;
constexpr size_t SMEM_USED = OFF_FLAG + 16;
constexpr size_t SMEM_BYTES = SMEM_USED + 1024;  // slack to align the base to 1024 bytes
static_assert(OFF_K % 1024 == 0 && OFF_V % 1024 == 0 && kTile % 1024 == 0,
              "swizzle atoms");
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");

struct ChunkParams {
  const uint16_t* q;
  float* out;
  float* lse;
  const int* block_table;
  const int* seq_lens;
  uint32_t* status;
  int B, Tq, Hq, Hkv, G, max_blocks, num_pages, max_seq_len;
  int range_begin, range_end;  // range_end > 0: restrict keys to [range_begin, range_end)
  int causal, n_shards, m_tiles;
  float qscale;  // softmax scale * log2(e)
};

// ---- tcgen05 / TMA wrappers -------------------------------------------------
// Shared-memory matrix descriptor, canonical 128B-swizzle layout: start address
// and the byte offsets between 8-row core groups (SBO) and between swizzle
// atoms along the leading dimension (LBO), all in 16-byte units; version 1;
// layout type 2 (128B swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for sm_100
  d |= (uint64_t)2 << 61;  // 128B swizzle
  return d;
}

// Instruction descriptor, kind::f16: fp32 accumulate, bf16 A and B, M = 128,
// N = 128; b_mn selects an MN-major B operand.
__host__ __device__ constexpr uint32_t instr_desc(bool b_mn) {
  return (1u << 4)                 // D format: f32
         | (1u << 7)               // A format: bf16
         | (1u << 10)              // B format: bf16
         | ((b_mn ? 1u : 0u) << 16)  // B major
         | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                         bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(da), "l"(db), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}

// The same with the A operand in TMEM (M rows = lanes, K along the columns).
__device__ __forceinline__ void mma_bf16_ts(uint32_t tmem_d, uint32_t tmem_a, uint64_t db,
                                            uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(tmem_d),
      "r"(tmem_a), "l"(db), "r"(idesc), "r"((uint32_t)accumulate)
      : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, "
      "%12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, "
      "%30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const float (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(__float_as_uint(v[0])), "r"(__float_as_uint(v[1])), "r"(__float_as_uint(v[2])),
      "r"(__float_as_uint(v[3])), "r"(__float_as_uint(v[4])), "r"(__float_as_uint(v[5])),
      "r"(__float_as_uint(v[6])), "r"(__float_as_uint(v[7])), "r"(__float_as_uint(v[8])),
      "r"(__float_as_uint(v[9])), "r"(__float_as_uint(v[10])), "r"(__float_as_uint(v[11])),
      "r"(__float_as_uint(v[12])), "r"(__float_as_uint(v[13])), "r"(__float_as_uint(v[14])),
      "r"(__float_as_uint(v[15])), "r"(__float_as_uint(v[16])), "r"(__float_as_uint(v[17])),
      "r"(__float_as_uint(v[18])), "r"(__float_as_uint(v[19])), "r"(__float_as_uint(v[20])),
      "r"(__float_as_uint(v[21])), "r"(__float_as_uint(v[22])), "r"(__float_as_uint(v[23])),
      "r"(__float_as_uint(v[24])), "r"(__float_as_uint(v[25])), "r"(__float_as_uint(v[26])),
      "r"(__float_as_uint(v[27])), "r"(__float_as_uint(v[28])), "r"(__float_as_uint(v[29])),
      "r"(__float_as_uint(v[30])), "r"(__float_as_uint(v[31]))
      : "memory");
}
// 32 consecutive 32-bit columns of this thread's TMEM lane, raw bits.
__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t (&v)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
      "%11, %12, %13, %14, %15, %16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, "
      "%29, %30, %31, %32};" ::"r"(taddr),
      "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
      "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]),
      "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]),
      "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]),
      "r"(v[29]), "r"(v[30]), "r"(v[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// 2-D TMA tile load (no multicast) completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
      "%3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// 2^x by the MUFU instruction (PTX ex2.approx, results below 2^-126 flush to 0)
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// byte offset of 16-byte chunk c (0..7) of row r inside a 128B-swizzled half
__device__ __forceinline__ uint32_t swz(int r, int c) {
  return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

__global__ void __launch_bounds__(kChunkThreads, 1)
    chunk_kernel(const ChunkParams p, const __grid_constant__ CUtensorMap tmK,
                 const __grid_constant__ CUtensorMap tmV) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem =
      smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);  // 1024-byte aligned base
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* k_full = bar;
  uint64_t* k_empty = bar + 2;
  uint64_t* v_full = bar + 4;
  uint64_t* v_empty = bar + 6;
  uint64_t* s_full = bar + 8;
  // [2]: every softmax thread has written its P row of the tiles with j & 1 == b
  // (one barrier per parity: Q K^T(j + 1) is issued before P V(j), so a warp can
  // reach tile j + 1 and arrive for it while another still works on tile j)
  uint64_t* p_full = bar + 10;
  uint64_t* o_done = bar + 12;  // [2]: P.V of tiles with j & 1 == b
  uint64_t* xbar = bar + 14;    // [4]: the two softmax warps of a TMEM lane quarter
  volatile float* xch = reinterpret_cast<volatile float*>(smem + OFF_XCH);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(smem + OFF_TMEM);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_FLAG);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tile = blockIdx.x % p.m_tiles, shard = blockIdx.x / p.m_tiles;
  const int kvh = blockIdx.y, b = blockIdx.z;

  // ---- key range of this CTA
  int L = p.seq_lens[b];
  if (L < 0 || L > p.max_seq_len) {
    if (threadIdx.x == 0 && m_tile == 0 && kvh == 0) dev_error(p.status, SKV_DEV_BAD_SEQLEN);
    L = 0;
  }
  int ra = 0, re = L;
  if (p.range_end > 0) {
    ra = max(p.range_begin, 0);
    re = min(p.range_end, L);
  }
  int k_lo = ra, k_hi = ra;  // this shard: [k_lo, k_hi)
  if (re > ra) {
    const long long span = re - ra;
    k_lo = ra + (int)(span * shard / p.n_shards);
    k_hi = ra + (int)(span * (shard + 1) / p.n_shards);
  }
  const int pos0 = (k_lo / kBlock) * kBlock;  // tiles start on a page
  const int n_tiles = (k_hi > k_lo) ? (k_hi - pos0 + BN - 1) / BN : 0;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&k_full[i], 1);   // producer arrival + transaction bytes
      mbar_init(&v_full[i], 1);
      mbar_init(&k_empty[i], 1);  // tcgen05.commit after the tile's Q K^T
      mbar_init(&v_empty[i], 1);  // tcgen05.commit after the tile's P V
    }
    mbar_init(&s_full[0], 1);    // tcgen05.commit after Q K^T
    mbar_init(&s_full[1], 1);
    mbar_init(&p_full[0], 256);  // every softmax thread has written its half P row
    mbar_init(&p_full[1], 256);
    mbar_init(&o_done[0], 1);    // tcgen05.commit after P V of even tiles
    mbar_init(&o_done[1], 1);    // ... and of odd tiles
    for (int i = 0; i < 4; ++i) mbar_init(&xbar[i], 2);  // one arrival per warp of the pair
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 1) {  // TMEM allocation (whole warp)
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32((const void*)tmem_slot)),
                 "r"(kTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // ---- Q rows -> shared memory (softmax threads, a half row each)
  const bool softmax_warp = warp >= 2 && warp < 10;
  const int srow = softmax_warp ? ((warp & 3) * 32 + lane) : -1;  // TMEM lane = row
  const int ch = (warp - 2) >> 2;                                // column half of this thread
  const int grow = m_tile * BM + srow;                          // row within the group
  const int t_row = (srow >= 0) ? grow / p.G : 0;
  const bool row_valid = srow >= 0 && t_row < p.Tq;
  if (srow >= 0) {
    uint4 chunks[8];
    if (row_valid) {
      const uint4* src = reinterpret_cast<const uint4*>(
          p.q + (((size_t)b * p.Tq + t_row) * p.Hq + (size_t)kvh * p.G + grow % p.G) * kHeadDim);
#pragma unroll
      for (int c = 0; c < 8; ++c) chunks[c] = src[ch * 8 + c];
    } else {
#pragma unroll
      for (int c = 0; c < 8; ++c) chunks[c] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int c = 0; c < 8; ++c)
      *reinterpret_cast<uint4*>(smem + OFF_Q + ch * kHalf + swz(srow, c)) = chunks[c];
    fence_async_smem();
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 || warp == 10) {
    // ------------------------------------------------------------ producers (K: warp 0, V: warp 10)
    const bool is_k = warp == 0;
    if (lane == 0 && n_tiles > 0) {
      const CUtensorMap* map = is_k ? &tmK : &tmV;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      unsigned char* ring = smem + (is_k ? OFF_K : OFF_V);
      asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
      const int* bt = p.block_table + (size_t)b * p.max_blocks;
      for (int j = 0; j < n_tiles; ++j) {
        const int st = j & 1;
        if (j >= 2 && !mbar_wait_bounded(&empty[st], ((j >> 1) - 1) & 1, abort_flag)) {
          dev_error(p.status, SKV_DEV_TIMEOUT);
          *abort_flag = 1;
          break;
        }
        int ys[2], nh = 0;
        for (int hh = 0; hh < 2; ++hh) {
          const int first = pos0 + j * BN + hh * kBlock;
          const int blk = first / kBlock;
          ys[hh] = -1;
          if (first >= k_hi || blk >= p.max_blocks) continue;
          const int page = bt[blk];
          if (page < 0 || page >= p.num_pages) {
            if (is_k) dev_error(p.status, SKV_DEV_BAD_PAGE);
            continue;
          }
          ys[hh] = (page * p.Hkv + kvh) * kBlock;
          ++nh;
        }
        unsigned char* dst = ring + (size_t)st * kTile;
        if (nh == 0) {
          mbar_arrive(&full[st]);
          continue;
        }
        mbar_arrive_expect_tx(&full[st], (uint32_t)nh * 2 * (kBlock * 64 * 2));
        for (int hh = 0; hh < 2; ++hh) {
          if (ys[hh] < 0) continue;
          for (int dh = 0; dh < 2; ++dh)
            tma_load_2d(dst + dh * kHalf + hh * (kHalf / 2), map, dh * 64, ys[hh], &full[st]);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0 && n_tiles > 0) {
      const uint32_t idesc_qk = instr_desc(false), idesc_pv = instr_desc(true);
      const uint32_t q_addr = smem_u32(smem + OFF_Q);
      auto issue_qk = [&](int j) -> bool {
        const int st = j & 1, sb = j & 1;
        // S buffer sb last held P(j - 2), read by a P.V issued before this Q K^T: the
        // tensor core runs them in order
        if (!mbar_wait_bounded(&k_full[st], (j >> 1) & 1, abort_flag)) return false;
        fence_after_sync();
        const uint32_t k_addr = smem_u32(smem + OFF_K + (size_t)st * kTile);
#pragma unroll
        for (int ks = 0; ks < kHeadDim / 16; ++ks) {
          const uint32_t off = (ks >> 2) * kHalf + (ks & 3) * 32;
          mma_bf16(tmem + sb * BN, smem_desc(q_addr + off, 16, 1024), smem_desc(k_addr + off, 16, 1024),
                   idesc_qk, ks > 0);
        }
        mma_commit(&s_full[sb]);
        mma_commit(&k_empty[st]);
        return true;
      };
      bool ok = issue_qk(0);
      for (int j = 0; ok && j < n_tiles; ++j) {
        if (j + 1 < n_tiles && !issue_qk(j + 1)) { ok = false; break; }
        if (!mbar_wait_bounded(&p_full[j & 1], (j >> 1) & 1, abort_flag)) { ok = false; break; }
        if (!mbar_wait_bounded(&v_full[j & 1], (j >> 1) & 1, abort_flag)) { ok = false; break; }
        fence_after_sync();
        const uint32_t v_addr = smem_u32(smem + OFF_V + (size_t)(j & 1) * kTile);
        const uint32_t pj = tmem + (uint32_t)(j & 1) * BN;
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks) {
          // A = P_h rows x 16 keys (TMEM, 8 columns of the half's S columns: the hi
          // terms, then the lo terms 32 columns on); B = V 16 keys x 128 dims
          // (MN-major); D = O_h
          const int h = ks >> 2, kk = ks & 3;
          const uint32_t b_off = ks * 16 * 128;
          const uint64_t dv = smem_desc(v_addr + b_off, kHalf, 1024);
          mma_bf16_ts(tmem + kColO + h * BM, pj + h * (BN / 2) + kk * 8, dv, idesc_pv, j > 0 || kk > 0);
          mma_bf16_ts(tmem + kColO + h * BM, pj + h * (BN / 2) + BN / 4 + kk * 8, dv, idesc_pv, true);
        }
        mma_commit(&o_done[j & 1]);
        mma_commit(&v_empty[j & 1]);
      }
      if (!ok) {
        dev_error(p.status, SKV_DEV_TIMEOUT);
        *abort_flag = 1;
      }
    }
  } else {
    // ------------------------------------------------------------ softmax
    constexpr int HC = BN / 2;                                       // keys of a half
    const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;  // TMEM lane field
    const uint32_t col_o = kColO + (uint32_t)ch * BM;               // this half's O_h
    const int q_pos = L - p.Tq + t_row;  // causal limit of this row
    float m_used = -INFINITY, l_sum = 0.f;
    bool o_live = false;  // O_h holds data (first P.V has run)
    bool ok = true;
    for (int j = 0; j < n_tiles && ok; ++j) {
      const int sb = j & 1;
      // every exit from this loop is taken by the whole warp (warp-wide tcgen05 below)
      if (!__all_sync(0xffffffffu, mbar_wait_bounded(&s_full[sb], (j >> 1) & 1, abort_flag))) {
        ok = false;
        break;
      }
      fence_after_sync();
      const uint32_t col_s = (uint32_t)sb * BN + (uint32_t)ch * HC;  // this half's S columns
      float s[HC];
#pragma unroll
      for (int c = 0; c < HC / 32; ++c) {
        float v[32];
        tmem_ld32(tmem + lane_base + col_s + c * 32, v);
#pragma unroll
        for (int i = 0; i < 32; ++i) s[c * 32 + i] = v[i];
      }
      tmem_wait_ld();
      // mask (boundary tiles only) and the max of the raw scores (the scale is
      // positive, so max(s) * scale is the max of the base-2 logits); 8 chains
      const int kp0 = pos0 + j * BN;
      const bool interior = row_valid && kp0 >= k_lo && kp0 + BN <= k_hi &&
                            (!p.causal || kp0 + BN - 1 <= q_pos);
      if (!interior) {
#pragma unroll
        for (int c = 0; c < HC; ++c) {
          const int kp = kp0 + ch * HC + c;
          bool valid = row_valid && kp >= k_lo && kp < k_hi;
          if (p.causal) valid = valid && kp <= q_pos;
          s[c] = valid ? s[c] : -INFINITY;
        }
      }
      float mx[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mx[u] = fmaxf(s[u], s[u + 8]);
#pragma unroll
      for (int c = 16; c < HC; c += 16)
#pragma unroll
        for (int u = 0; u < 8; ++u) mx[u] = fmaxf(mx[u], fmaxf(s[c + u], s[c + 8 + u]));
      const float tmax = p.qscale * fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                          fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      // Lazy rescale: only when the max grows by more than 2^8.  The decision is
      // taken for the whole warp (tcgen05.ld / st are warp-wide instructions and
      // must not sit in divergent code): if any row of the warp needs it, every
      // row moves to max(m_used, tmax), which is exact for all of them.
      if (__any_sync(0xffffffffu, tmax > m_used + 8.f)) {
        const float m_new = fmaxf(m_used, tmax);
        // 0 when m_used is -inf; 1 for a row whose max did not grow (and for a
        // row that has seen no key yet, m_used = m_new = -inf)
        const float alpha = (m_new == m_used) ? 1.f : exp2f(m_used - m_new);
        l_sum *= alpha;
        if (o_live) {  // O_h must hold every P.V so far: wait for the one of tile j - 1
          const int jp = j - 1;
          const bool got = mbar_wait_bounded(&o_done[jp & 1], (jp >> 1) & 1, abort_flag);
          if (!__all_sync(0xffffffffu, got)) {
            ok = false;
            break;
          }
          fence_after_sync();
#pragma unroll
          for (int c = 0; c < BM / 32; ++c) {
            float v[32];
            tmem_ld32(tmem + lane_base + col_o + c * 32, v);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= alpha;
            tmem_st32(tmem + lane_base + col_o + c * 32, v);
          }
          tmem_wait_st();
        }
        m_used = m_new;
      }
      const float mu = (m_used == -INFINITY) ? 0.f : m_used;
      // P_h = 2^(s * scale - m_h), split into two bf16 terms P_h = hi + lo
      // (hi = bf16(p), lo = bf16(p - hi)): hi as bf16 pairs over the first 32 of
      // this half's S columns, lo over the other 32 (all already read).  P.V runs
      // on both, so the weights enter the product with a relative error of about
      // 2^-16 instead of bf16's 2^-8.  Packed fp32x2 for the exponent argument
      // and for l, which sums the unrounded values.
      const f2 sc2 = pack2(p.qscale, p.qscale), nm2 = pack2(-mu, -mu);
      f2 ls2[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) ls2[u] = pack2(0.f, 0.f);
      uint32_t pw[HC / 2], pl[HC / 2];
#pragma unroll
      for (int c8 = 0; c8 < HC / 8; ++c8) {
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          f2 x = nm2;
          ffma2(x, pack2(s[c8 * 8 + 2 * u], s[c8 * 8 + 2 * u + 1]), sc2);
          float x0, x1;
          unpack2(x, x0, x1);
          const float p0 = ex2(x0), p1 = ex2(x1);
          const f2 pp = pack2(p0, p1);
          ls2[u] = fadd2(ls2[u], pp);
          const __nv_bfloat162 h2 = __floats2bfloat162_rn(p0, p1);  // p0 in the low half
          const uint32_t hw = *reinterpret_cast<const uint32_t*>(&h2);
          pw[c8 * 4 + u] = hw;
          f2 rem = pp;
          ffma2(rem, bf2_to_f2(hw), pack2(-1.f, -1.f));  // p - hi, exact in fp32
          float r0, r1;
          unpack2(rem, r0, r1);
          const __nv_bfloat162 l2 = __floats2bfloat162_rn(r0, r1);
          pl[c8 * 4 + u] = *reinterpret_cast<const uint32_t*>(&l2);
        }
      }
      tmem_st32u(tmem + lane_base + col_s, pw);
      tmem_st32u(tmem + lane_base + col_s + HC / 2, pl);
      tmem_wait_st();
      {
        const f2 t2 = fadd2(fadd2(ls2[0], ls2[1]), fadd2(ls2[2], ls2[3]));
        float a0, a1;
        unpack2(t2, a0, a1);
        l_sum += a0 + a1;
      }
      // keys outside the range on a boundary tile: zero their V rows (they may hold
      // anything) so that 0 * V stays 0; each thread clears its half of the row
      const int key = kp0 + srow;
      if (kp0 < k_lo || kp0 + BN > k_hi) {
        // V(j) must have landed before its rows are cleared (v_full cannot run two
        // phases ahead: its next phase needs the P.V of this tile)
        if (!__all_sync(0xffffffffu, mbar_wait_bounded(&v_full[j & 1], (j >> 1) & 1, abort_flag))) {
          ok = false;
          break;
        }
        if (key < k_lo || key >= k_hi) {
          unsigned char* sV = smem + OFF_V + (size_t)(j & 1) * kTile;
#pragma unroll
          for (int c = 0; c < 8; ++c)
            *reinterpret_cast<uint4*>(sV + ch * kHalf + swz(srow, c)) = make_uint4(0u, 0u, 0u, 0u);
        }
      }
      fence_async_smem();
      fence_before_sync();
      mbar_arrive(&p_full[j & 1]);
      o_live = true;
    }
    // ---- epilogue: combine the two halves' (m, l, O) of this row
    if (ok && n_tiles > 0) {  // the last P.V (the tensor core runs them in order)
      const int jl = n_tiles - 1;
      if (!mbar_wait_bounded(&o_done[jl & 1], (jl >> 1) & 1, abort_flag)) ok = false;
    }
    float m_o = -INFINITY, l_o = 0.f;  // the other half's
    {
      xch[(0 * 2 + ch) * BM + srow] = m_used;
      xch[(1 * 2 + ch) * BM + srow] = l_sum;
      __syncwarp();
      mbar_arrive_if(&xbar[warp & 3], lane == 0);
      if (!mbar_wait_bounded(&xbar[warp & 3], 0, abort_flag)) ok = false;
      m_o = xch[(0 * 2 + (ch ^ 1)) * BM + srow];
      l_o = xch[(1 * 2 + (ch ^ 1)) * BM + srow];
    }
    if (!ok) {
      dev_error(p.status, SKV_DEV_TIMEOUT);
      *abort_flag = 1;
    }
    fence_after_sync();
    // weights of O_0 and O_1 (this thread's half is O_ch, the other O_(ch^1))
    const float M = fmaxf(m_used, m_o);
    const float w_me = (l_sum > 0.f) ? exp2f(m_used - M) : 0.f;
    const float w_ot = (l_o > 0.f) ? exp2f(m_o - M) : 0.f;
    const float Lt = l_sum * w_me + l_o * w_ot;
    const float w0 = ch == 0 ? w_me : w_ot, w1 = ch == 0 ? w_ot : w_me;
    // this thread writes output dims ch*64 .. ch*64+63 from both accumulators
    float o[HC];
    if (n_tiles > 0) {
#pragma unroll
      for (int c = 0; c < HC / 32; ++c) {
        float v0[32], v1[32];
        tmem_ld32(tmem + lane_base + kColO + ch * HC + c * 32, v0);
        tmem_ld32(tmem + lane_base + kColO + BM + ch * HC + c * 32, v1);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) o[c * 32 + i] = v0[i] * w0 + v1[i] * w1;
      }
    }
    if (row_valid) {
      const float inv = (Lt > 0.f) ? 1.f / Lt : 0.f;
      const size_t rows = (size_t)p.B * p.Tq * p.Hq;
      const size_t row = ((size_t)b * p.Tq + t_row) * p.Hq + (size_t)kvh * p.G + grow % p.G;
      float4* dst = reinterpret_cast<float4*>(p.out + ((size_t)shard * rows + row) * kHeadDim + ch * HC);
#pragma unroll
      for (int c = 0; c < HC / 4; ++c) {
        if (n_tiles > 0)
          dst[c] = make_float4(o[4 * c] * inv, o[4 * c + 1] * inv, o[4 * c + 2] * inv, o[4 * c + 3] * inv);
        else
          dst[c] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (ch == 0)
        p.lse[(size_t)shard * rows + row] =
            (Lt > 0.f) ? (M + log2f(Lt)) * 0.6931471805599453f : -INFINITY;
    }
  }
  // ---- teardown: every tcgen05 operation is complete; free TMEM
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols)
                 : "memory");
  }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (no -lcuda).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  }
  return fn;
}

// Pool [rows = pages * Hkv * 64][128] bf16 as a 2-D tensor, boxes of 64 rows x 64 columns
// (128 bytes) landing 128B-swizzled.
bool make_pool_map(CUtensorMap* m, const void* pool, long long rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
  const cuuint32_t box[2] = {64, 64};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(pool), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int launch_chunk(const DecodeParams& dp, int Tq, int causal, int n_shards, void* stream) {
  CUtensorMap tk, tv;
  const long long rows = (long long)dp.num_pages * dp.Hkv * kBlock;
  if (!make_pool_map(&tk, dp.k_pool, rows) || !make_pool_map(&tv, dp.v_pool, rows))
    return (int)cudaErrorInvalidValue;
  ChunkParams p{};
  p.q = dp.q;
  p.out = dp.out;
  p.lse = dp.lse;
  p.block_table = dp.block_table;
  p.seq_lens = dp.seq_lens;
  p.status = dp.status;
  p.B = dp.B;
  p.Tq = Tq;
  p.Hq = dp.Hq;
  p.Hkv = dp.Hkv;
  p.G = dp.Hq / dp.Hkv;
  p.max_blocks = dp.max_blocks;
  p.num_pages = dp.num_pages;
  p.max_seq_len = dp.max_seq_len;
  p.range_begin = dp.range_begin;
  p.range_end = dp.range_end;
  p.causal = causal;
  p.n_shards = n_shards < 1 ? 1 : n_shards;
  p.m_tiles = (Tq * p.G + BM - 1) / BM;
  p.qscale = dp.qscale;
  static std::atomic<bool> attr_set[64];  // per device; racing first calls only repeat the set-up
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return (int)cudaErrorInvalidDevice;
  if (!attr_set[dev]) {
    cudaError_t e =
        cudaFuncSetAttribute(chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES);
    if (e != cudaSuccess) return (int)e;
    attr_set[dev] = true;
  }
  dim3 grid(p.m_tiles * p.n_shards, p.Hkv, p.B);
  chunk_kernel<<<grid, kChunkThreads, SMEM_BYTES, static_cast<cudaStream_t>(stream)>>>(p, tk, tv);
  return (int)cudaGetLastError();
}

}  // namespace skv
