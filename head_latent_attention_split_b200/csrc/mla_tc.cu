// Tensor-core (tcgen05 + TMA) absorbed-MLA decode for r = 512, d_r = 64, 64-token
// cache blocks, bf16 queries, bf16 or FP8 e4m3 (per-token scale) cache.
//
// Design (one CTA pair = one cluster of 2 per worker and row group):
//  * The 128 query rows of a row group (Sq * H rows of one sequence, zero-padded) are
//    the M = 128 rows of every MMA. Their fp32 output O[128 x 512] would fill all 512
//    TMEM columns, so the two CTAs of the pair split the latent channels: CTA j owns
//    latent channels [256 j, 256 j + 256) and RoPE channels [32 j, 32 j + 32) of every
//    MMA, for all 128 rows.
//  * TMEM per CTA (128 lanes = query rows): O [0, 256), partial scores S [256, 320),
//    probabilities P (bf16 pairs, double buffered) [320, 384), and the CTA's half of
//    the absorbed query, latent part, as a TMEM A operand [384, 512).
//  * Each CTA TMA-loads only its channel slice of every 64-token cache block
//    (4 x [64 tok][64 ch] 128B-swizzled + [64 tok][32 ch] 64B-swizzled = 36 KB per
//    stage, 4 stages). The query's RoPE part stays in shared memory (8 KB).
//  * QK: S_j[128 x 64] = Q_j . C_j^T over the CTA's 288 channels (16 MMAs with A in
//    TMEM + 2 with A in shared memory, K = 16 each). The full score is S_0 + S_1.
//  * Row split of the softmax: in every TMEM lane quarter q, lanes [32 q + 16 j, +16)
//    hold CTA j's own rows and the other 16 lanes the peer's, read and written with the
//    16-lane TMEM shape. Warp q (0-3) works on the own lanes of quarter q, warp q + 4 on
//    the peer lanes, so both kinds of work spread over the four SM sub-partitions, and a
//    row's 64 columns live in one warp (threads t and t + 16). Per tile:
//      - the peer-lane warps stage those rows of S_j (fp32) and move each quarter to the
//        peer with one bulk copy (bytes complete on the peer's mbarrier);
//      - the own-lane warps add the peer's partials to theirs, take the row maximum (a
//        shuffle), the exponentials (each once, in the row's owner) and the row sums,
//        write P into TMEM and send the same bf16 rows plus one rescale factor per row
//        back the same way;
//      - the peer-lane warps write the received P rows into their TMEM lanes and
//        rescale those O rows when the owner moved a maximum. They serve their two
//        streams (ship scores, take probabilities) as an event loop.
//    24.25 KB cross the pair per tile and direction. The running maximum only moves
//    when a tile raises it by more than 2^8, so O is rescaled rarely.
//  * PV: O_j[128 x 256] += P[128 x 64] . C_j[64 x 256] with A = P from TMEM and B =
//    the SAME shared-memory tile the QK used, read N-major (4 MMAs, N = 256). The MMA
//    issuer runs QK(k) then PV(k - 2).
//  * FP8 cache, exact: c_t = code_t * s_t with a per-token fp32 scale s_t. The
//    producer TMA-loads the CTA's 256 e4m3 codes per token (16 KB) into the upper half
//    of the stage, the bf16 RoPE key into its slot and the block's 64 scales; two
//    converter warps (one token row per thread) write the codes back as bf16 in place
//    (every e4m3 value is exact in bf16) in the 128B-swizzled layout the bf16 path
//    loads, and replace the RoPE key by kR_t / s_t split into bf16 hi + lo parts
//    (2^-16 relative). The score MMAs then give S_t / s_t; the softmax multiplies each
//    column by s_t, and P by s_t before PV (sum_t p_t s_t code_t = sum_t p_t c_t), with
//    the row sum over the unscaled p_t.
//  * Warp roles: warps 0-3 own-lane softmax and epilogue, warps 4-7 peer-lane exchange
//    and epilogue, warp 8 TMA producer, warp 9 TMEM allocator and single-thread MMA
//    issuer, warps 10-11 FP8 converters (sparse decode: warp 10 is a second copy warp);
//    mbarrier pipelines between them. Every wait is bounded (timeout -> MLA_ERR_TIMEOUT,
//    clean exit).
//  * Sparse decode (DeepSeek Sparse Attention: "TransMLA & Sparse Latent Attention"
//    lesson, Chapter 7 "DSA runs in MLA's MQA mode"): the same kernel over each
//    sequence's list of selected positions instead of its whole length. The per-sequence
//    length is the list's count, and tile t holds list entries [64 t, 64 t + 64). Two
//    copy warps (8 and 10, on different SM sub-partitions, 32 rows each) map them through
//    the block table and copy the token rows of the CTA's channel slice with 16-byte
//    cp.async copies (one 512-byte row slice per warp instruction) into the same swizzled
//    stage layout; each lane's copies complete one arrival on the stage barrier. Entries
//    past the count are zero-filled without a read. The copies go through the LSU rather
//    than TMA row gathers (four rows per load), which measured slower on B200.
// The work split over workers (CTA pairs) is the flat block list plan of mla_device.cuh.
#include <cuda.h>
#include <cuda_fp16.h>

#include <cmath>
#include <mutex>

#include "mla_device.cuh"
#include "mla_tc.h"
#include "ptx_sm100.cuh"

namespace mla {
namespace {

using namespace ptx;

constexpr int kR = 512, kDR = 64, kBS = 64;
constexpr int kRows = 128;           // query rows per row group = MMA M
constexpr int kStages = 4;

// shared memory layout, byte offsets from a 1024-aligned base
constexpr uint32_t kKvLatChunk = kBS * 128;                      // [64 tok][64 ch] bf16, 128B swizzle
constexpr uint32_t kKvRope = kBS * 64;                           // [64 tok][32 ch] bf16, 64B swizzle
constexpr uint32_t kQRope = kRows * 64;                          // [128 rows][32 ch] bf16, 64B swizzle
// Exchange buffers. Partial scores of 64 rows: 4 regions of [32 rows][32 cols] fp32;
// probabilities of 64 rows: 4 regions of [32 rows][32 tokens] bf16 followed by 64 fp32
// rescale factors. Each CTA stages what it sends in a buffer laid out like the peer's
// receive buffer and moves every warp's region with one bulk copy.
constexpr uint32_t kRxSRegion = 32 * 32 * 4;
constexpr uint32_t kRxSBytes = 4 * kRxSRegion;                   // 16 KB
constexpr uint32_t kRxPRegion = 32 * 32 * 2;
constexpr uint32_t kRxPAlpha = 4 * kRxPRegion;                   // offset of the rescale factors
constexpr uint32_t kRxPBytes = kRxPAlpha + 64 * 4;               // 8448
constexpr uint32_t kLrxBytes = 64 * 4;                           // the peer's row sums of its rows
constexpr uint32_t kCtlBytes = 4096;
// bf16 stage: latent chunks + RoPE. FP8 stage: latent chunks + RoPE hi + RoPE lo + scales.
template <bool kFp8> struct Geo {
  static constexpr uint32_t kStageBytes = kFp8 ? 41984u : 36864u;
  static constexpr uint32_t kOffRopeLo = 4 * kKvLatChunk + kKvRope;   // FP8 only
  static constexpr uint32_t kOffScale = kOffRopeLo + kKvRope;         // FP8 only: 64 fp32
  static constexpr uint32_t kOffKv = 0;
  static constexpr uint32_t kOffQr = kStages * kStageBytes;
  static constexpr uint32_t kRxSBufs = kFp8 ? 1 : 2;             // receive buffers for partial scores
  static constexpr uint32_t kOffRxS = kOffQr + kQRope;
  static constexpr uint32_t kOffRxP = kOffRxS + kRxSBufs * kRxSBytes;   // one receive buffer for P
  static constexpr uint32_t kOffTxS = kOffRxP + kRxPBytes;             // staging of outgoing scores
  static constexpr uint32_t kOffTxP = kOffTxS + kRxSBytes;             // ... and probabilities
  static constexpr uint32_t kOffCtl = kOffTxP + kRxPBytes;
  static constexpr uint32_t kSmemBytes = kOffCtl + kCtlBytes + 1024;   // + alignment slack
};
static_assert(Geo<true>::kOffScale + 256 <= Geo<true>::kStageBytes && Geo<true>::kStageBytes % 1024 == 0, "fp8 stage");
static_assert(Geo<false>::kOffScale == Geo<true>::kOffScale, "one stage geometry for both caches");
static_assert(Geo<false>::kOffQr % 1024 == 0 && Geo<true>::kOffQr % 1024 == 0, "buffers need 1024-byte alignment");
static_assert(Geo<false>::kSmemBytes <= 232448 && Geo<true>::kSmemBytes <= 232448, "shared memory budget");
static_assert(kRxPBytes % 16 == 0 && Geo<true>::kOffTxS % 16 == 0 && Geo<false>::kOffTxS % 16 == 0,
              "bulk copies need 16-byte alignment");

// TMEM columns (32-bit lanes x columns; lane = query row)
constexpr uint32_t kTmemO = 0;       // 256: this CTA's output channels
constexpr uint32_t kTmemS = 256;     // 64: partial scores of the current tile
constexpr uint32_t kTmemP = 320;     // 2 x 32: probabilities, bf16 pairs
constexpr uint32_t kTmemQ = 384;     // 128: absorbed query, this CTA's 256 latent channels
constexpr uint32_t kTmemCols = 512;

constexpr int kSoftmaxThreads = 256;  // warps 0-7
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kConvWarp0 = 10;        // FP8 cache: warps 10-11 decode codes in place; sparse: warp 10 copies
constexpr int kConvThreads = 64;      // one thread per token row of a tile
template <bool kFp8, bool kSparse>
constexpr int threads_for() { return kFp8 ? 384 : kSparse ? 352 : 320; }
constexpr uint32_t kFp8CodeBytes = kBS * 256;                    // this CTA's codes of one block
constexpr uint32_t kFp8StageTx = kFp8CodeBytes + kKvRope + kBS * 4;   // codes, RoPE key, scales

constexpr float kRescaleThreshold = 8.0f;   // log2 units: rescale O only if the max grows > 2^8
// FP8 cache: the RoPE key is divided by max(s_t, 2^-64) and the score column multiplied by the
// same factor. For s_t >= 2^-64 that is exact; below it (an all-zero latent stores s_t = 0, and
// 1 / s_t would overflow for tiny scales) the latent term picks up an error of at most
// 2^-64 * |q . code|, far below any tolerance, instead of inf * 0 = NaN.
constexpr float kScaleFloor = 0x1p-64f;

struct Ctl {
  uint64_t kv_full[kStages];
  uint64_t kv_empty[kStages];
  uint64_t kv_ready[kStages];   // FP8: the converted bf16 tile is in place
  uint64_t cv_loaded[kStages];  // FP8: every converter thread holds its codes in registers
  uint64_t q_full, q_empty;
  uint64_t s_full, s_empty;
  uint64_t p_full[2];       // P of tile t (both row halves) is in TMEM slot t & 1, O rescaled
  uint64_t pv_done[2];      // PV of tile t completes a phase of pv_done[t & 1]
  uint64_t rxs_full[2];     // the peer's partial scores of tile t landed in buffer t % kRxSBufs
  uint64_t rxp_full;        // the peer's probabilities and rescale factors of the next tile landed
  uint64_t txs_ok[2];       // the peer has read the partial scores we last sent into its buffer b
  uint64_t txp_ok;          // ... the probabilities
  uint64_t lrx_full[2];     // the peer's row sums of segment s, s & 1 == b, have landed
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  WorkerPlan plan;
  float lrx[2][64];         // [segment parity][peer's own row]: written by the peer
};
static_assert(sizeof(Ctl) <= kCtlBytes, "control block too large");

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// e4m3 pair (low byte = first code) -> f16x2, exact (every e4m3 value is an f16 value)
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t two_codes) {
  uint32_t h2;
  asm("{\n\t.reg .b16 c;\n\tcvt.u16.u32 c, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, c;\n\t}" : "=r"(h2) : "r"(two_codes));
  return h2;
}

// 16-byte global -> shared copy that bypasses L1 (LDGSTS). src_bytes = 0 reads nothing and
// writes 16 zero bytes.
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(src_bytes) : "memory");
}
// One arrival on the mbarrier once every cp.async this thread issued before has completed
// (noinc: the arrival counts against the barrier's expected count).
__device__ __forceinline__ void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

template <bool kFp8, bool kSparse>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(threads_for<kFp8, kSparse>(), 1)
    tc_decode_kernel(const __grid_constant__ CUtensorMap tm_qr, const __grid_constant__ CUtensorMap tm_kv,
                     const __grid_constant__ CUtensorMap tm_kr, const __grid_constant__ CUtensorMap tm_sc,
                     const DecodeArgs a, const int n_rg, const uint64_t timeout_ns, const uint64_t drain_ns) {
  using G = Geo<kFp8>;
  constexpr uint32_t kStageBytes = G::kStageBytes;
  constexpr uint32_t kOffKv = G::kOffKv;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem + G::kOffCtl);
  const uint32_t sKv = smem_u32(smem + kOffKv);
  const uint32_t sQr = smem_u32(smem + G::kOffQr);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int cluster = (int)(blockIdx.x >> 1);
  const int w = cluster / n_rg, rg = cluster % n_rg;
  const int cap = a.len_cap;
  volatile int* abort = &ctl.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&ctl.kv_full[i]), kSparse ? 64 : 1);   // sparse: one cp.async arrival per copy lane
      mbar_init(smem_u32(&ctl.kv_empty[i]), 1);
    }
    mbar_init(smem_u32(&ctl.q_full), 1 + kSoftmaxThreads);   // RoPE part by TMA + latent part into TMEM
    mbar_init(smem_u32(&ctl.q_empty), 1);
    mbar_init(smem_u32(&ctl.s_full), 1);
    mbar_init(smem_u32(&ctl.s_empty), kSoftmaxThreads);
    for (int i = 0; i < 2; ++i) mbar_init(smem_u32(&ctl.p_full[i]), kSoftmaxThreads);
    for (int i = 0; i < 2; ++i) mbar_init(smem_u32(&ctl.pv_done[i]), 1);
    for (int i = 0; i < 2; ++i) {
      // receive barriers: one local arrival plus the peer's bytes; armed for tiles (segments) 0 and 1
      mbar_init(smem_u32(&ctl.rxs_full[i]), 1);
      mbar_arrive_expect_tx(smem_u32(&ctl.rxs_full[i]), kRxSBytes);
      mbar_init(smem_u32(&ctl.lrx_full[i]), 1);
      mbar_arrive_expect_tx(smem_u32(&ctl.lrx_full[i]), kLrxBytes);
      mbar_init(smem_u32(&ctl.txs_ok[i]), 4);   // one arrival per consuming warp of the peer
    }
    for (int i = 0; i < kStages; ++i) {
      mbar_init(smem_u32(&ctl.kv_ready[i]), kConvThreads);
      mbar_init(smem_u32(&ctl.cv_loaded[i]), kConvThreads);
    }
    mbar_init(smem_u32(&ctl.rxp_full), 1);
    mbar_arrive_expect_tx(smem_u32(&ctl.rxp_full), kRxPBytes);   // armed for tile 0
    mbar_init(smem_u32(&ctl.txp_ok), 4);
    mbar_init(smem_u32(&ctl.drain), 1);
    ctl.abort = 0;
    fence_mbarrier_init_cluster();
  }
  if (warp == kProducerWarp) {
    const WorkerPlan p = warp_plan(a.seq_lens, a.B, a.bs, cap, a.W, w, a.status);
    if (lane == 0) {
      ctl.plan = p;
      prefetch_tmap(&tm_qr);
      prefetch_tmap(&tm_kv);
      prefetch_tmap(&tm_kr);
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&ctl.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();          // barriers of both CTAs initialised, TMEM allocated, plan ready
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;
  const WorkerPlan plan = ctl.plan;

  if (kSparse && (warp == kProducerWarp || warp == kConvWarp0)) {
    // ------------------------------------------------------------------ copy producers (sparse)
    // Two warps on different SM sub-partitions; warp 8 also loads the query. Warp h takes
    // rows [32 h, 32 h + 32) of every tile: its lanes map those listed positions to cache
    // rows (-1 = no row), then the whole warp copies each row with 16-byte cp.async copies
    // into the same swizzled stage layout the TMA path writes: lane l takes unit l of the
    // row's 512-byte latent slice (one row per warp instruction), and one 16-byte unit of
    // four rows' 64-byte RoPE slices. Every lane's copies of a tile complete one arrival on
    // the stage barrier; rows that are not there are zero-filled without a read.
    const int half = warp == kProducerWarp ? 0 : 1;
    SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
    Segment sg;
    uint32_t g = 0, seg = 0;
    bool ok = true;
    const char* cache = static_cast<const char*>(a.cache);
    constexpr uint32_t kRowBytes = (kR + kDR) * 2;
    const uint32_t lat_src = 512 * rank + 16 * lane;                  // byte offset in a cache row
    const uint32_t lat_dst = (lane >> 3) * kKvLatChunk;               // 64-channel chunk of the unit
    const uint32_t rope_src = 2 * kR + 64 * rank + 16 * (lane & 3);
    while (ok && it.next(sg)) {
      if (half == 0 && lane == 0) {
        ok = mbar_wait<false>(smem_u32(&ctl.q_empty), (seg & 1) ^ 1, abort, timeout_ns);
        if (ok) {
          const uint32_t qbar = smem_u32(&ctl.q_full);
          mbar_arrive_expect_tx(qbar, kQRope);
          tma_load_3d(sQr, &tm_qr, qbar, 32 * rank, rg * kRows, sg.b);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      for (int tile = sg.tile_begin; tile < sg.tile_end; ++tile, ++g) {
        int rw = -1;
        {
          const int j = tile * kBS + 32 * half + lane;   // list entry
          if (j < sg.Lc) {
            const int t = __ldg(a.sel_idx + (size_t)sg.b * a.top_k + j);
            const int blk = (t >= 0 && t < a.max_blocks * kBS) ? __ldg(a.block_table + (size_t)sg.b * a.max_blocks + t / kBS) : -1;
            if (blk >= 0 && blk < a.num_blocks)
              rw = blk * kBS + t % kBS;
            else
              set_status(a.status, MLA_ERR_BAD_BLOCK_ID);
          }
        }
        const uint32_t st = g % kStages, ph = (g / kStages) & 1;
        if (lane == 0) ok = mbar_wait<false>(smem_u32(&ctl.kv_empty[st]), ph ^ 1, abort, timeout_ns);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        const uint32_t base = sKv + st * kStageBytes;
#pragma unroll 8
        for (int ii = 0; ii < 32; ++ii) {
          const int i = 32 * half + ii;
          const int row = __shfl_sync(0xffffffffu, rw, ii);
          const char* src = cache + (size_t)(row < 0 ? 0 : row) * kRowBytes + lat_src;
          cp_async_16(base + lat_dst + i * 128 + (((lane & 7) ^ (i & 7)) << 4), src, row < 0 ? 0u : 16u);
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const int ii = 8 * k + (lane >> 2);                // rows 8k .. 8k + 7 of the half, four lanes each
          const int i = 32 * half + ii;
          const int row = __shfl_sync(0xffffffffu, rw, ii);
          const char* src = cache + (size_t)(row < 0 ? 0 : row) * kRowBytes + rope_src;
          cp_async_16(base + 4 * kKvLatChunk + i * 64 + (((lane & 3) ^ ((i >> 1) & 3)) << 4), src, row < 0 ? 0u : 16u);
        }
        cp_async_arrive_noinc(smem_u32(&ctl.kv_full[st]));
      }
      ++seg;
    }
    // Each lane waits for its own copies, so nothing lands after the CTA exits. (A stage
    // barrier is no drain signal here: after a timeout one copy warp may have arrived on it
    // and the other not.)
    cp_async_wait_all();
    if (lane == 0 && !ok) set_status(a.status, MLA_ERR_TIMEOUT);
  } else if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
      Segment sg;
      uint32_t g = 0, seg = 0;
      bool ok = true;
      while (ok && it.next(sg)) {
        ok = mbar_wait<false>(smem_u32(&ctl.q_empty), (seg & 1) ^ 1, abort, timeout_ns);
        if (!ok) break;
        const uint32_t qbar = smem_u32(&ctl.q_full);
        mbar_arrive_expect_tx(qbar, kQRope);
        tma_load_3d(sQr, &tm_qr, qbar, 32 * rank, rg * kRows, sg.b);
        for (int tile = sg.tile_begin; tile < sg.tile_end; ++tile, ++g) {
          const uint32_t st = g % kStages, ph = (g / kStages) & 1;
          ok = mbar_wait<false>(smem_u32(&ctl.kv_empty[st]), ph ^ 1, abort, timeout_ns);
          if (!ok) break;
          const int blk = checked_block(a.block_table, a.max_blocks, sg.b, tile, a.num_blocks, a.status);
          const uint32_t bar = smem_u32(&ctl.kv_full[st]);
          const uint32_t base = sKv + st * kStageBytes;
          if constexpr (kFp8) {
            // codes [64 tok][256 B] into the upper half of the latent area, RoPE key into its slot
            mbar_arrive_expect_tx(bar, kFp8StageTx);
            tma_load_3d(base + 2 * kKvLatChunk, &tm_kv, bar, 256 * rank, 0, blk);
            tma_load_3d(base + 4 * kKvLatChunk, &tm_kr, bar, 32 * rank, 0, blk);
            tma_load_3d(base + Geo<kFp8>::kOffScale, &tm_sc, bar, 0, 0, blk);
          } else {
            mbar_arrive_expect_tx(bar, kStageBytes);
            for (int c = 0; c < 4; ++c) tma_load_3d(base + c * kKvLatChunk, &tm_kv, bar, 256 * rank + 64 * c, 0, blk);
            tma_load_3d(base + 4 * kKvLatChunk, &tm_kr, bar, kR + 32 * rank, 0, blk);
          }
        }
        ++seg;
      }
      // let every load already issued land before the CTA can exit
      int dummy = 0;
      for (uint32_t i = 0; i < kStages && i < g; ++i) {
        const uint32_t gl = g - 1 - i;   // the latest load of stage gl % kStages
        mbar_wait<false>(smem_u32(&ctl.kv_full[gl % kStages]), (gl / kStages) & 1, &dummy, drain_ns);
      }
      if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // FP8 cache: the latent score MMAs and the PV run on fp16 operands (codes and P in fp16),
      // the RoPE MMAs stay bf16
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, 64, false);
      constexpr uint32_t idesc_qk_lat = kFp8 ? idesc_f16_f32(128, 64, false) : idesc_qk;
      constexpr uint32_t idesc_pv = kFp8 ? idesc_f16_f32(128, 256, true) : idesc_bf16_f32(128, 256, true);
      SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
      Segment sg;
      uint32_t g = 0, seg = 0;
      bool ok = true;
      auto issue_pv = [&](uint32_t gp, bool first) -> bool {
        const uint32_t st = gp % kStages, pb = gp & 1;
        if (!mbar_wait<false>(smem_u32(&ctl.p_full[pb]), (gp >> 1) & 1, abort, timeout_ns)) return false;
        tc_fence_after();
        const uint32_t base = sKv + st * kStageBytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          // B = C[16 tokens][256 channels], channels contiguous (N-major): 64-channel
          // groups 8 KB apart (LBO), 8-token groups 1 KB apart (SBO)
          const uint64_t bdesc = smem_desc(base + kk * 2048, kKvLatChunk, 1024, kSwizzle128B);
          mma_ts(tmem + kTmemO, tmem + kTmemP + 32 * pb + 8 * kk, bdesc, idesc_pv, (first && kk == 0) ? 0u : 1u);
        }
        mma_commit(smem_u32(&ctl.kv_empty[st]));
        mma_commit(smem_u32(&ctl.pv_done[pb]));
        return true;
      };
      while (ok && it.next(sg)) {
        ok = mbar_wait<false>(smem_u32(&ctl.q_full), seg & 1, abort, timeout_ns);
        if (!ok) break;
        tc_fence_after();
        const uint32_t g0 = g;
        const int n = sg.tile_end - sg.tile_begin;
        for (int li = 0; li < n; ++li, ++g) {
          const uint32_t st = g % kStages;
          ok = mbar_wait<false>(smem_u32(kFp8 ? &ctl.kv_ready[st] : &ctl.kv_full[st]), (g / kStages) & 1, abort,
                                timeout_ns) &&
               mbar_wait<false>(smem_u32(&ctl.s_empty), (g & 1) ^ 1, abort, timeout_ns);
          if (!ok) break;
          tc_fence_after();
          if constexpr (kSparse) fence_proxy_async_smem();   // the tile was written by cp.async
          const uint32_t base = sKv + st * kStageBytes;
          const uint32_t d = tmem + kTmemS;
#pragma unroll
          for (int kk = 0; kk < 16; ++kk) {
            // latent channels [16 kk, 16 kk + 16): A = Q from TMEM, B = the cache chunk
            const uint64_t bdesc = smem_desc(base + (kk >> 2) * kKvLatChunk + (kk & 3) * 32, 16, 1024, kSwizzle128B);
            mma_ts(d, tmem + kTmemQ + 8 * kk, bdesc, idesc_qk_lat, kk ? 1u : 0u);
          }
#pragma unroll
          for (int kk = 0; kk < (kFp8 ? 4 : 2); ++kk) {
            // RoPE channels; FP8: k-steps 2, 3 repeat the query against the lo parts
            const uint64_t adesc = smem_desc(sQr + (kk & 1) * 32, 16, 512, kSwizzle64B);
            const uint64_t bdesc =
                smem_desc(base + (kk < 2 ? 4 * kKvLatChunk : Geo<kFp8>::kOffRopeLo) + (kk & 1) * 32, 16, 512,
                          kSwizzle64B);
            mma_ss(d, adesc, bdesc, idesc_qk, 1u);
          }
          mma_commit(smem_u32(&ctl.s_full));
          if (li == n - 1) mma_commit(smem_u32(&ctl.q_empty));
          if (li >= 2) {
            ok = issue_pv(g - 2, li == 2);
            if (!ok) break;
          }
        }
        if (!ok) break;
        for (int li = n >= 2 ? n - 2 : 0; ok && li < n; ++li) ok = issue_pv(g0 + li, li == 0);
        ++seg;
      }
      // every MMA issued so far completes before TMEM can be released
      int dummy = 0;
      mma_commit(smem_u32(&ctl.drain));
      mbar_wait<false>(smem_u32(&ctl.drain), 0, &dummy, drain_ns);
      if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
    }
  } else if (warp >= kConvWarp0) {
    // ------------------------------------------------------------------ FP8 converters
    if constexpr (kFp8) {
      const int tok = threadIdx.x - kConvWarp0 * 32;     // token row of the tile, 0..63
      SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
      Segment sg;
      uint32_t g = 0;
      bool ok = true;
      while (ok && it.next(sg)) {
        for (int tile = sg.tile_begin; tile < sg.tile_end; ++tile, ++g) {
          const uint32_t st = g % kStages, ph = (g / kStages) & 1;
          ok = __all_sync(0xffffffffu, mbar_wait<false>(smem_u32(&ctl.kv_full[st]), ph, abort, timeout_ns));
          if (!ok) break;
          uint8_t* base = smem + kOffKv + st * kStageBytes;
          const float sc = *reinterpret_cast<const float*>(base + Geo<kFp8>::kOffScale + tok * 4);   // TMA'd
          // RoPE key / scale as bf16 hi + lo (its 64-byte row, 64B-swizzled, in place + lo slot)
          {
            const float inv_sc = 1.0f / fmaxf(sc, kScaleFloor);
            uint8_t* hi_row = base + 4 * kKvLatChunk + tok * 64;
            uint8_t* lo_row = base + Geo<kFp8>::kOffRopeLo + tok * 64;
#pragma unroll
            for (int pc = 0; pc < 4; ++pc) {
              const int phys = (pc ^ ((tok >> 1) & 3)) << 4;
              const uint4 v = *reinterpret_cast<const uint4*>(hi_row + phys);
              const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
              uint32_t h[4], l[4];
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const float x0 = __uint_as_float(wv[j] << 16) * inv_sc;
                const float x1 = __uint_as_float(wv[j] & 0xFFFF0000u) * inv_sc;
                h[j] = pack_bf16x2(x0, x1);
                l[j] = pack_bf16x2(x0 - __uint_as_float(h[j] << 16), x1 - __uint_as_float(h[j] & 0xFFFF0000u));
              }
              *reinterpret_cast<uint4*>(hi_row + phys) = make_uint4(h[0], h[1], h[2], h[3]);
              *reinterpret_cast<uint4*>(lo_row + phys) = make_uint4(l[0], l[1], l[2], l[3]);
            }
          }
          // codes of this token -> fp16 (the latent MMAs' B operand): 16 pieces of 16 bytes
          // (channels [16 p, 16 p + 16)). Piece
          // order is XOR-staggered by the token so that a warp's loads hit distinct banks.
          const uint8_t* src = base + 2 * kKvLatChunk + tok * 256;
          auto convert_piece = [&](const uint4 v, const int p) {
            // -> channels [16 p, 16 p + 16): chunk p / 4, 16-byte pieces 2 (p % 4) and
            // 2 (p % 4) + 1 of the 128B-swizzled row
            const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
            uint32_t o[8];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              o[2 * j] = e4m3x2_to_f16x2(wv[j] & 0xFFFFu);   // exact: e4m3 values are f16 values
              o[2 * j + 1] = e4m3x2_to_f16x2(wv[j] >> 16);
            }
            uint8_t* row = base + (p >> 2) * kKvLatChunk + tok * 128;
            const int p0 = 2 * (p & 3);
            *reinterpret_cast<uint4*>(row + (((p0) ^ (tok & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
            *reinterpret_cast<uint4*>(row + (((p0 + 1) ^ (tok & 7)) << 4)) = make_uint4(o[4], o[5], o[6], o[7]);
          };
          // pieces 8-15 live where chunks 2-3 will be written: hold them in registers
          uint4 upper[8];
#pragma unroll
          for (int j = 0; j < 8; ++j) upper[j] = *reinterpret_cast<const uint4*>(src + ((8 + (j ^ (tok & 7))) << 4));
          // pieces 0-7 convert straight into chunks 0-1 (which hold no codes)
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const int pc = j ^ (tok & 7);
            convert_piece(*reinterpret_cast<const uint4*>(src + (pc << 4)), pc);
          }
          // every row's upper codes are in registers before any row's bf16 lands on them
          mbar_arrive(smem_u32(&ctl.cv_loaded[st]));
          ok = __all_sync(0xffffffffu, mbar_wait<false>(smem_u32(&ctl.cv_loaded[st]), ph, abort, timeout_ns));
          if (!ok) break;
#pragma unroll
          for (int j = 0; j < 8; ++j) convert_piece(upper[j], 8 + (j ^ (tok & 7)));
          fence_proxy_async_smem();
          mbar_arrive(smem_u32(&ctl.kv_ready[st]));
        }
      }
      if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
    }
  } else {
    // ------------------------------------------------------------------ softmax, exchange, epilogue
    // Row split: in every TMEM lane quarter q, lanes [32 q + 16 rank, +16) hold this CTA's own
    // rows and the other 16 lanes the peer's. Warp q (0-3) works on the own lanes of quarter
    // q, warp q + 4 on the peer lanes, so both kinds of work spread over the four SM
    // sub-partitions. With the 16-lane TMEM access shape, thread t and t + 16 share row
    // t & 15 of the warp's lanes: columns [0, 32) and [32, 64) of a tile.
    const int quad = warp & 3;
    const bool own = warp < 4;
    const int rr = lane & 15;                           // row within the warp's 16 lanes
    const int hf = lane >> 4;                           // column half of the tile / of O
    const int lbase = quad * 32 + 16 * (own ? (int)rank : (int)peer);
    const uint32_t lane_off = (uint32_t)lbase << 16;
    const int row = lbase + rr;                         // TMEM lane = query row in the group
    const int orow = quad * 16 + rr;                    // the row among the 64 its owner normalises
    const bool leader = lane == 0 && quad == 0;         // one thread per role re-arms
    constexpr uint32_t kNbS = G::kRxSBufs;
    // Exchange regions: quarter q of every buffer holds 16 rows; a row is 64 fp32 scores
    // (256 B) or 64 bf16 probabilities (128 B). Own warp q of one CTA and peer warp q + 4
    // of the other fill / drain region q. 16-byte pieces of a row are XOR-swizzled by the
    // row so that 8 consecutive rows hit distinct banks.
    const uint32_t s_row = quad * kRxSRegion + rr * 256;
    const uint32_t p_row = quad * kRxPRegion + rr * 128;
    auto piece = [&](int c) { return (uint32_t)((c ^ (rr & 7)) << 4); };
    const uint32_t rxs = smem_u32(smem + G::kOffRxS), txs = smem_u32(smem + G::kOffTxS);
    const uint32_t rxp = smem_u32(smem + G::kOffRxP), txp = smem_u32(smem + G::kOffTxP);
    const uint32_t alpha_off = kRxPAlpha + orow * 4;
    const int grow = rg * kRows + row;
    const bool valid_row = grow < a.rows;
    const int s_idx = valid_row ? grow / a.H : 0;
    const float scale_log2 = a.scale_log2;
    SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
    Segment sg;
    uint32_t g = 0, seg = 0;
    bool ok = true;
    // waits of this role are made warp-uniform: tcgen05.ld/st below are warp-collective
    auto wait_local = [&](uint32_t bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait<false>(bar, parity, abort, timeout_ns));
    };
    auto wait_peer = [&](uint32_t bar, uint32_t parity) {
      return __all_sync(0xffffffffu, mbar_wait<true>(bar, parity, abort, timeout_ns));
    };
    // lane 0 waits for a barrier the peer arrives on (a buffer handed back); the warp follows
    auto wait_remote_arrival = [&](uint32_t bar, uint32_t parity) {
      bool r = true;
      if (lane == 0) r = mbar_wait<false>(bar, parity, abort, timeout_ns);
      return __all_sync(0xffffffffu, r);
    };
    // PV(j) done. Valid while PV(j - 2) is complete and PV(j + 2) cannot be (its P is
    // not written yet): callers only wait for PVs of the current segment, in order.
    auto wait_pv = [&](uint32_t j) { return wait_local(smem_u32(&ctl.pv_done[j & 1]), (j >> 1) & 1); };
    // O row of this thread (columns [128 hf, +128) of the CTA's 256) times alpha; all
    // earlier PVs complete
    auto rescale_o = [&](float alpha) {
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t v[16];
        const uint32_t ta = tmem + lane_off + kTmemO + 16 * c;
        tmem_ld16x2<128>(ta, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
        tmem_st16x2<128>(ta, v);
      }
      tmem_wait_st();
    };
    // this thread's 32 partial-score columns of the current tile, out of TMEM
    auto load_s = [&](uint32_t gt, uint32_t* sv) {
      if (!wait_local(smem_u32(&ctl.s_full), gt & 1)) return false;
      tc_fence_after();
      tmem_ld16x2<32>(tmem + lane_off + kTmemS, sv);
      tmem_ld16x2<32>(tmem + lane_off + kTmemS + 16, sv + 16);
      tmem_wait_ld();
      tc_fence_before();
      mbar_arrive(smem_u32(&ctl.s_empty));
      return true;
    };
    while (it.next(sg)) {
      bool written = false;   // this segment's rows of out / partials written
      do {
      if (!ok) break;
      // this segment's absorbed query, latent half of this CTA, into TMEM (the warp's 16 rows)
      ok = wait_local(smem_u32(&ctl.q_empty), (seg & 1) ^ 1);
      if (!ok) break;
      {
        uint32_t qv[64];
        const uint4* src = reinterpret_cast<const uint4*>((const uint16_t*)a.q_lat +
                                                         ((size_t)sg.b * a.rows + (valid_row ? grow : 0)) * kR +
                                                         256 * rank + 128 * hf);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const uint4 v = valid_row ? __ldg(src + i) : make_uint4(0u, 0u, 0u, 0u);
          qv[4 * i] = v.x;
          qv[4 * i + 1] = v.y;
          qv[4 * i + 2] = v.z;
          qv[4 * i + 3] = v.w;
        }
        if constexpr (kFp8) {
          // the latent score MMAs take fp16 operands: the bf16 query words to fp16 (exact for
          // |q| in [2^-14, 65504] with at most 8 significant bits; smaller values lose bits)
#pragma unroll
          for (int i = 0; i < 64; ++i)
            qv[i] = pack_f16x2(__uint_as_float(qv[i] << 16), __uint_as_float(qv[i] & 0xFFFF0000u));
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) tmem_st16x2<64>(tmem + lane_off + kTmemQ + 16 * c, qv + 16 * c);
        tmem_wait_st();
        tc_fence_before();
        mbar_arrive(smem_u32(&ctl.q_full));
      }
      const int n = sg.tile_end - sg.tile_begin;
      const int last_tile = (sg.Lc + kBS - 1) / kBS - 1;
      float m_run = -INFINITY, l_run = 0.f;   // own rows: running maximum (log2 units), this thread's sum
      if (own) {
        int n_row = valid_row ? (a.causal ? sg.Lc - a.Sq + 1 + s_idx : sg.Lc) : 0;
        if (n_row < 0) n_row = 0;
        for (int li = 0; li < n; ++li) {
          const uint32_t gt = g + li, b = gt & 1;
          const int tile = sg.tile_begin + li;
          uint32_t sv[32];
          ok = load_s(gt, sv);
          if (!ok) break;
          // ---- the peer's partials of our rows; full scores; row maximum
          const uint32_t bs = gt % kNbS;
          ok = wait_peer(smem_u32(&ctl.rxs_full[bs]), (gt / kNbS) & 1);
          if (!ok) break;
          const uint32_t rx = rxs + bs * kRxSBytes + s_row;
          float x[32];
          float mh = -INFINITY;
          const int valid = min(max(n_row - tile * kBS - 32 * hf, 0), 32);   // of my 32 columns
          const float4* cs = nullptr;   // FP8: token scales of my columns
          if constexpr (kFp8) {
            const uint32_t stg = gt % kStages;
            ok = wait_local(smem_u32(&ctl.kv_ready[stg]), (gt / kStages) & 1);
            if (!ok) break;
            cs = reinterpret_cast<const float4*>(smem + kOffKv + stg * kStageBytes + G::kOffScale + 128 * hf);
          }
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            uint4 v;
            asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(rx + piece(8 * hf + c)));
            const float r4[4] = {__uint_as_float(v.x), __uint_as_float(v.y), __uint_as_float(v.z),
                                 __uint_as_float(v.w)};
            float c4[4] = {1.f, 1.f, 1.f, 1.f};
            if constexpr (kFp8) {
              const float4 t = cs[c];
              c4[0] = fmaxf(t.x, kScaleFloor);
              c4[1] = fmaxf(t.y, kScaleFloor);
              c4[2] = fmaxf(t.z, kScaleFloor);
              c4[3] = fmaxf(t.w, kScaleFloor);
            }
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const int k = 4 * c + i;
              const float sc = (__uint_as_float(sv[k]) + r4[i]) * c4[i] * scale_log2;
              x[k] = k < valid ? sc : -INFINITY;
              mh = fmaxf(mh, x[k]);
            }
          }
          const float mt = fmaxf(mh, __shfl_xor_sync(0xffffffffu, mh, 16));   // depends on every value read
          __syncwarp();
          // the peer may refill our region of buffer bs (tile gt + kNbS)
          if (lane == 0) mbar_arrive_remote_cta(mapa(smem_u32(&ctl.txs_ok[bs]), peer));
          if (leader) mbar_arrive_expect_tx(smem_u32(&ctl.rxs_full[bs]), kRxSBytes);
          // ---- exponentials, P into TMEM and to the peer
          const bool grow_max = mt > m_run + kRescaleThreshold;
          const bool rescale = grow_max && m_run != -INFINITY;
          const float alpha = rescale ? ex2_approx(m_run - mt) : 1.f;
          // P slot b is free once PV(gt - 2) has completed
          if (li >= 2) {
            ok = wait_pv(gt - 2);
            if (!ok) break;
          }
          if (__any_sync(0xffffffffu, rescale)) {
            // O holds this segment's tiles before gt: wait for the last PV, then scale
            if (li >= 1) {
              ok = wait_pv(gt - 1);
              if (!ok) break;
            }
            tc_fence_after();
            rescale_o(alpha);
          }
          if (grow_max) {
            l_run *= alpha;
            m_run = mt;
          }
          uint32_t pk[16];
          float psum = 0.f;
          const bool any = m_run != -INFINITY;
          float pcs[32];     // FP8: P columns carry the token scale into PV (0 for unseen tokens)
          if constexpr (kFp8) {
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const float4 v = cs[c];
              pcs[4 * c] = 4 * c < valid ? v.x : 0.f;
              pcs[4 * c + 1] = 4 * c + 1 < valid ? v.y : 0.f;
              pcs[4 * c + 2] = 4 * c + 2 < valid ? v.z : 0.f;
              pcs[4 * c + 3] = 4 * c + 3 < valid ? v.w : 0.f;
            }
          }
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float p0 = any ? ex2_approx(x[k] - m_run) : 0.f;
            const float p1 = any ? ex2_approx(x[k + 1] - m_run) : 0.f;
            psum += p0 + p1;
            if constexpr (kFp8)
              pk[k >> 1] = pack_f16x2(p0 * pcs[k], p1 * pcs[k + 1]);   // the PV's fp16 A operand
            else
              pk[k >> 1] = pack_bf16x2(p0, p1);
          }
          l_run += psum;
          tmem_st16x2<16>(tmem + lane_off + kTmemP + 32 * b, pk);
          // stage the P row (and the rescale factor) like the peer's receive buffer; our
          // previous copy out of the staging region must have finished reading it
          if (lane == 0) bulk_wait_group_read<0>();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 4; ++c)
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(txp + p_row + piece(4 * hf + c)),
                         "r"(pk[4 * c]), "r"(pk[4 * c + 1]), "r"(pk[4 * c + 2]), "r"(pk[4 * c + 3])
                         : "memory");
          if (hf == 0)
            asm volatile("st.shared.f32 [%0], %1;" ::"r"(txp + alpha_off), "f"(alpha) : "memory");
          fence_proxy_async_smem();
          // the peer's receive buffer is free once it has read tile gt - 1
          if (gt >= 1) {
            ok = wait_remote_arrival(smem_u32(&ctl.txp_ok), (gt - 1) & 1);
            if (!ok) break;
          }
          __syncwarp();
          if (lane == 0) {
            const uint32_t bar = mapa(smem_u32(&ctl.rxp_full), peer);
            bulk_copy_to_peer(mapa(rxp + quad * kRxPRegion, peer), txp + quad * kRxPRegion, kRxPRegion, bar);
            bulk_copy_to_peer(mapa(rxp + kRxPAlpha + quad * 64, peer), txp + kRxPAlpha + quad * 64, 64, bar);
            bulk_commit_group();
          }
          // Slots past the sequence end in its last block may hold anything (NaN): zero
          // those token rows of this CTA's latent slice before the PV reads them.
          const int tail = sg.Lc % kBS;
          if (tile == last_tile && tail != 0) {
            const uint32_t stg = gt % kStages;
            ok = wait_local(smem_u32(kFp8 ? &ctl.kv_ready[stg] : &ctl.kv_full[stg]), (gt / kStages) & 1);
            if (!ok) break;
            uint8_t* base = smem + kOffKv + stg * kStageBytes;
            const int per_chunk = (kBS - tail) * 8;          // 16-byte pieces per chunk
            for (int i = threadIdx.x; i < 4 * per_chunk; i += 128) {   // the 4 own warps
              const int chunk = i / per_chunk, rem = i % per_chunk;
              *reinterpret_cast<uint4*>(base + chunk * kKvLatChunk + (tail + rem / 8) * 128 + (rem % 8) * 16) =
                  make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
          }
          tmem_wait_st();
          tc_fence_before();
          mbar_arrive(smem_u32(&ctl.p_full[b]));
        }
      } else {
        // Peer lanes: two in-order streams served as they become ready -- ship the partial
        // scores of each tile to the peer, and take the peer's P rows of each tile into
        // TMEM. Lane 0 polls, the warp follows its choice.
        int ship = 0, recv = 0;   // next segment-local tile of each stream
        uint32_t spins = 0;
        uint64_t t_idle = 0;
        while (recv < n) {
          int act = 0;
          if (lane == 0) {
            if (ship < n && mbar_test_wait(smem_u32(&ctl.s_full), (g + ship) & 1))
              act = 1;
            else if (recv < ship && mbar_test_wait_cluster(smem_u32(&ctl.rxp_full), (g + recv) & 1))
              act = 2;
            else if ((++spins & 255u) == 0u) {
              const uint64_t now = globaltimer();
              if (*abort) act = 3;
              else if (t_idle == 0) t_idle = now;
              else if (now - t_idle > timeout_ns) { *abort = 1; act = 3; }
            }
            if (act == 1 || act == 2) { spins = 0; t_idle = 0; }
          }
          act = __shfl_sync(0xffffffffu, act, 0);
          if (act == 3) { ok = false; break; }
          if (act == 1) {
            const uint32_t gt = g + ship, bs = gt % kNbS;
            uint32_t sv[32];
            ok = load_s(gt, sv);
            if (!ok) break;
            // stage the rows; our previous copy out of the staging region must be done reading
            if (lane == 0) bulk_wait_group_read<0>();
            __syncwarp();
#pragma unroll
            for (int c = 0; c < 8; ++c)
              asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(txs + s_row + piece(8 * hf + c)),
                           "r"(sv[4 * c]), "r"(sv[4 * c + 1]), "r"(sv[4 * c + 2]), "r"(sv[4 * c + 3])
                           : "memory");
            fence_proxy_async_smem();
            // the peer's receive buffer bs is free once it has read tile gt - kNbS
            if (gt >= kNbS) {
              ok = wait_remote_arrival(smem_u32(&ctl.txs_ok[bs]), ((gt / kNbS) + 1) & 1);
              if (!ok) break;
            }
            __syncwarp();
            if (lane == 0) {
              bulk_copy_to_peer(mapa(rxs + bs * kRxSBytes + quad * kRxSRegion, peer), txs + quad * kRxSRegion,
                                kRxSRegion, mapa(smem_u32(&ctl.rxs_full[bs]), peer));
              bulk_commit_group();
            }
            ++ship;
          } else if (act == 2) {
            const uint32_t gp = g + recv, b = gp & 1;
            ok = wait_peer(smem_u32(&ctl.rxp_full), gp & 1);   // completes at once
            if (!ok) break;
            uint32_t pk[16];
#pragma unroll
            for (int c = 0; c < 4; ++c)
              asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(pk[4 * c]), "=r"(pk[4 * c + 1]), "=r"(pk[4 * c + 2]), "=r"(pk[4 * c + 3])
                           : "r"(rxp + p_row + piece(4 * hf + c)));
            float alpha;
            asm volatile("ld.shared.f32 %0, [%1];" : "=f"(alpha) : "r"(rxp + alpha_off));
            if (recv >= 2) {   // P slot b held tile gp - 2 of this segment
              ok = wait_pv(gp - 2);
              if (!ok) break;
            }
            if (__any_sync(0xffffffffu, alpha != 1.f)) {
              if (recv >= 1) {
                ok = wait_pv(gp - 1);
                if (!ok) break;
              }
              tc_fence_after();
              rescale_o(alpha);
            }
            tmem_st16x2<16>(tmem + lane_off + kTmemP + 32 * b, pk);   // consumes the loaded rows
            __syncwarp();
            if (lane == 0) mbar_arrive_remote_cta(mapa(smem_u32(&ctl.txp_ok), peer));
            if (leader) mbar_arrive_expect_tx(smem_u32(&ctl.rxp_full), kRxPBytes);   // tile gp + 1
            tmem_wait_st();
            tc_fence_before();
            mbar_arrive(smem_u32(&ctl.p_full[b]));
            ++recv;
          }
        }
      }
      if (!ok) break;
      g += n;

      // epilogue: O / l -> out (single split) or the normalised partial (several splits).
      // PVs up to g - 3 were waited for above; wait for the last two in order.
      for (uint32_t j = (n >= 2 ? g - 2 : g - 1); ok && j < g; ++j) ok = wait_pv(j);
      if (!ok) break;
      tc_fence_after();
      float l_tot;
      if (own) {
        l_tot = l_run + __shfl_xor_sync(0xffffffffu, l_run, 16);
        if (hf == 0)
          st_async_b32(mapa(smem_u32(&ctl.lrx[seg & 1][orow]), peer), __float_as_uint(l_tot),
                       mapa(smem_u32(&ctl.lrx_full[seg & 1]), peer));
      } else {
        ok = wait_peer(smem_u32(&ctl.lrx_full[seg & 1]), (seg >> 1) & 1);
        if (!ok) break;
        l_tot = ctl.lrx[seg & 1][orow];
        __syncwarp();
        if (leader) mbar_arrive_expect_tx(smem_u32(&ctl.lrx_full[seg & 1]), kLrxBytes);   // segment seg + 2
      }
      const bool poisoned = segment_poisoned(a, sg.b, sg.tile_begin, sg.tile_end);
      const float inv = poisoned ? __uint_as_float(0x7FC00000u) : l_tot > 0.f ? 1.f / l_tot : 0.f;
      const size_t qrow = (size_t)sg.b * a.rows + grow;
      const bool direct = sg.splits == 1;
      const size_t prow = (size_t)(w + sg.b) * a.rows + grow;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {
        uint32_t v[16];
        tmem_ld16x2<128>(tmem + lane_off + kTmemO + 16 * c, v);
        tmem_wait_ld();
        if (!valid_row) continue;
        const int ch = 256 * (int)rank + 128 * hf + 16 * c;
        if (direct && a.out_dtype == kBF16) {
          uint4 o0, o1;
          o0.x = pack_bf16x2(__uint_as_float(v[0]) * inv, __uint_as_float(v[1]) * inv);
          o0.y = pack_bf16x2(__uint_as_float(v[2]) * inv, __uint_as_float(v[3]) * inv);
          o0.z = pack_bf16x2(__uint_as_float(v[4]) * inv, __uint_as_float(v[5]) * inv);
          o0.w = pack_bf16x2(__uint_as_float(v[6]) * inv, __uint_as_float(v[7]) * inv);
          o1.x = pack_bf16x2(__uint_as_float(v[8]) * inv, __uint_as_float(v[9]) * inv);
          o1.y = pack_bf16x2(__uint_as_float(v[10]) * inv, __uint_as_float(v[11]) * inv);
          o1.z = pack_bf16x2(__uint_as_float(v[12]) * inv, __uint_as_float(v[13]) * inv);
          o1.w = pack_bf16x2(__uint_as_float(v[14]) * inv, __uint_as_float(v[15]) * inv);
          uint4* dst = reinterpret_cast<uint4*>((uint16_t*)a.out + qrow * kR + ch);
          dst[0] = o0;
          dst[1] = o1;
        } else {
          float* dst = direct ? (float*)a.out + qrow * kR + ch : a.o_part + prow * kR + ch;
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(dst + i) =
                make_float4(__uint_as_float(v[i]) * inv, __uint_as_float(v[i + 1]) * inv,
                            __uint_as_float(v[i + 2]) * inv, __uint_as_float(v[i + 3]) * inv);
        }
      }
      if (own && hf == 0 && valid_row) {
        const float lse_v = poisoned ? __uint_as_float(0x7FC00000u)
                            : l_tot > 0.f ? (m_run + log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
        if (direct)
          a.lse[qrow] = lse_v;
        else
          a.lse_part[prow] = lse_v;
      }
      if (sg.split == 0 && rg == 0 && rank == 0 && threadIdx.x == 0) {
        a.meta[2 * sg.b] = sg.first_worker;
        a.meta[2 * sg.b + 1] = sg.splits;
      }
      tc_fence_before();
      ++seg;
      written = true;
      } while (0);
      if (!written && valid_row) {
        // a wait ran out: this CTA's channels of the segment's rows (and the lse) become NaN
        const float qnan = __uint_as_float(0x7FC00000u);
        const bool direct = sg.splits == 1;
        const size_t qrow = (size_t)sg.b * a.rows + grow, prow = (size_t)(w + sg.b) * a.rows + grow;
        for (int k = 0; k < 128; ++k) {
          const int ch = 256 * (int)rank + 128 * hf + k;
          if (direct && a.out_dtype == kBF16)
            ((uint16_t*)a.out)[qrow * kR + ch] = 0x7FC0;
          else
            (direct ? (float*)a.out + qrow * kR : a.o_part + prow * kR)[ch] = qnan;
        }
        if (own && hf == 0) (direct ? a.lse[qrow] : a.lse_part[prow]) = qnan;
      }
    }
    if (lane == 0) bulk_wait_group_read<0>();   // staging regions stay valid until read
    if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  cluster_sync();   // no CTA leaves while its peer may still touch its shared memory
}

// ---------------------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = (EncodeTiledFn)p;
  });
  return fn;
}

// 3-D tensor map: dims (inner -> outer), byte strides of dims 1 and 2, box.
bool make_map_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1,
                 uint64_t s2, uint32_t b0, uint32_t b1, CUtensorMapSwizzle sw,
                 CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {s1, s2};
  const cuuint32_t box[3] = {b0, b1, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int row_groups(int rows) { return (rows + kRows - 1) / kRows; }

}  // namespace

bool tc_supported(int r, int d_r, int block_size, int q_dtype, int cache_dtype, int out_dtype, int rows) {
  return r == kR && d_r == kDR && block_size == kBS && q_dtype == kBF16 &&
         (cache_dtype == kBF16 || cache_dtype == kE4M3) &&
         (out_dtype == kBF16 || out_dtype == kF32) && rows >= 1 && row_groups(rows) <= 1024;
}

int tc_auto_workers(int sms, int rows) {
  const int w = sms / (2 * row_groups(rows));
  return w > 0 ? w : 1;
}

bool tc_workers_ok(int W, int rows) { return W >= 1 && (long long)W * row_groups(rows) * 2 <= 65535; }

cudaError_t launch_tc_decode(const DecodeArgs& a, cudaStream_t s) {
  const int n_rg = row_groups(a.rows);
  CUtensorMap tqr, tkv, tkr, tsc;
  const uint64_t rows = (uint64_t)a.rows;
  const bool fp8 = a.cache_dtype == kE4M3;
  const bool sparse = a.sel_idx != nullptr;
  if (sparse && (fp8 || a.Sq != 1 || a.causal)) return cudaErrorInvalidValue;
  bool ok = make_map_3d(&tqr, a.q_rope, kDR, rows, a.B, kDR * 2, rows * kDR * 2, 32, kRows, CU_TENSOR_MAP_SWIZZLE_64B);
  if (sparse) {
    tkv = tkr = tqr;   // the sparse kernel copies cache rows with cp.async; no cache maps
  } else if (fp8) {
    // codes [num_blocks][64][512] e4m3 (256-byte boxes, no swizzle), RoPE keys [num_blocks][64][64] bf16
    ok = ok &&
         make_map_3d(&tkv, a.cache, kR, kBS, a.num_blocks, kR, (uint64_t)kBS * kR, 256, kBS, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_DATA_TYPE_UINT8) &&
         make_map_3d(&tkr, a.k_rope, kDR, kBS, a.num_blocks, kDR * 2, (uint64_t)kBS * kDR * 2, 32, kBS,
                     CU_TENSOR_MAP_SWIZZLE_64B) &&
         make_map_3d(&tsc, a.kv_scale, kBS, 1, a.num_blocks, kBS * 4, kBS * 4, kBS, 1, CU_TENSOR_MAP_SWIZZLE_NONE,
                     CU_TENSOR_MAP_DATA_TYPE_FLOAT32);
  } else {
    ok = ok &&
         make_map_3d(&tkv, a.cache, kR + kDR, kBS, a.num_blocks, (kR + kDR) * 2, (uint64_t)kBS * (kR + kDR) * 2, 64,
                     kBS, CU_TENSOR_MAP_SWIZZLE_128B) &&
         make_map_3d(&tkr, a.cache, kR + kDR, kBS, a.num_blocks, (kR + kDR) * 2, (uint64_t)kBS * (kR + kDR) * 2, 32,
                     kBS, CU_TENSOR_MAP_SWIZZLE_64B);
  }
  if (!ok) return cudaErrorInvalidValue;
  if (!fp8) tsc = tkr;   // unused by the bf16 kernels
  static std::once_flag attr_once[3][64];
  int dev = 0;
  cudaGetDevice(&dev);
  const int variant = sparse ? 2 : fp8 ? 1 : 0;
  cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once[variant][dev & 63], [&] {
    attr_err = variant == 1 ? cudaFuncSetAttribute(tc_decode_kernel<true, false>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, Geo<true>::kSmemBytes)
               : variant == 2 ? cudaFuncSetAttribute(tc_decode_kernel<false, true>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, Geo<false>::kSmemBytes)
                              : cudaFuncSetAttribute(tc_decode_kernel<false, false>,
                                                     cudaFuncAttributeMaxDynamicSharedMemorySize, Geo<false>::kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const uint64_t timeout_ns = wait_timeout_ns(), drain_ns = drain_timeout_ns();
  const dim3 grid(2 * a.W * n_rg);
  if (variant == 1)
    tc_decode_kernel<true, false><<<grid, threads_for<true, false>(), Geo<true>::kSmemBytes, s>>>(tqr, tkv, tkr, tsc, a, n_rg,
                                                                                           timeout_ns, drain_ns);
  else if (variant == 2)
    tc_decode_kernel<false, true><<<grid, threads_for<false, true>(), Geo<false>::kSmemBytes, s>>>(tqr, tkv, tkr, tsc, a,
                                                                                             n_rg, timeout_ns, drain_ns);
  else
    tc_decode_kernel<false, false><<<grid, threads_for<false, false>(), Geo<false>::kSmemBytes, s>>>(tqr, tkv, tkr, tsc, a,
                                                                                              n_rg, timeout_ns, drain_ns);
  return cudaGetLastError();
}

}  // namespace mla
