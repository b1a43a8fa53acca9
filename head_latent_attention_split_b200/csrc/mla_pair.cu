// Split-role tensor-core (tcgen05 + TMA) absorbed-MLA decode for r = 512, d_r = 64, 64-token
// cache blocks, bf16 queries and a bf16 cache; dense token ranges, or (kSparse) each sequence's
// list of selected positions.
//
// The fp32 output of 128 query rows over all 512 latent channels, O[128 x 512], fills the 512
// TMEM columns of one SM, so a decode worker is a cluster of two CTAs. The roles differ:
//
//   score CTA (cluster rank 0): streams every tile of the worker's range whole (512 latent +
//     64 RoPE channels) and computes full scores S = Q . C^T with tcgen05: A = the absorbed
//     query held in TMEM, B = the cache rows in shared memory. Tiles are scored two at a time
//     (N = 128 tokens per MMA): on B200 a tcgen05 MMA costs ~60 cycles up to N = 64 and ~70 at
//     N = 128, so pairs of tiles nearly double the score rate. The cache ring is 3 slots of
//     48 KB, each three 64-channel chunks of both tiles of a pair (6 TMA boxes per barrier).
//     Eight softmax warps (two per SM sub-partition: warp q takes the first tile's 64 columns
//     of rows [32q, 32q + 32), warp q + 4 the second tile's) run the online softmax in
//     registers, thread = query row, share the row maximum through shared memory, and write
//     each tile's message (bf16 P[128 x 64] as K-major core matrices plus one rescale factor
//     and 1/row-sum per row, 17 KB) into one of four staging buffers; a post warp sends each
//     message with one bulk copy into the output CTA's shared memory.
//   output CTA (cluster rank 1): streams the same tiles' 512 latent channels (one 4-D TMA box per
//     256 channels; the second read of each tile is served by L2), rescales O rows whose
//     running maximum moved, and accumulates O[128 x 512] += P . C with tcgen05 (A = P in
//     shared memory, B = the tile read N-major, N = 256), then normalises O into the output
//     (or the split partial).
//
// Only P crosses between the SMs, in one direction. The completion of the PV that read a
// receive buffer is signalled straight to the score CTA by the tensor core (a commit arriving on
// the score CTA's barrier), and the output CTA hands a staging buffer back with one remote
// arrive once its message has landed, so no thread waits on a round trip per tile.
//
// The running maximum of a row only moves when a tile pair raises it by more than 2^8 (log2
// units), so O is rescaled rarely; the softmax uses base-2 exponentials of scale * log2(e) *
// score. Work split over workers: the flat block-list plan of mla_device.cuh (same as every
// kernel); pairs never straddle two sequences (a sequence with an odd number of tiles ends with
// a single tile, scored with N = 64). Every wait is bounded; a timeout sets MLA_ERR_TIMEOUT and
// the rows of the unfinished segments are written as NaN.
#include <cuda.h>

#include <cmath>
#include <mutex>

#include "mla_device.cuh"
#include "mla_tc.h"
#include "ptx_sm100.cuh"

namespace mla {
namespace {

using namespace ptx;

constexpr int kR = 512, kDR = 64, kBS = 64, kRows = 128;
constexpr uint32_t kChunk = kBS * 128;                 // [64 tok][64 ch] bf16, 128-byte swizzle
constexpr uint32_t kDChunk = 2 * kChunk;               // one chunk of both tiles of a pair
constexpr int kChunksS = 9;                            // score CTA: 8 latent chunks + the RoPE chunk
constexpr int kGroupS = 3;                             // score CTA: double chunks per ring slot (6 boxes)
constexpr uint32_t kSlotBytesS = kGroupS * kDChunk;    // 48 KB
constexpr int kSlotsS = 3;                             // score CTA ring of slots
constexpr uint32_t kHalf = 4 * kChunk;                 // output CTA half stage: 256 channels of a tile
constexpr int kHalvesO = 5;                            // output CTA ring of half stages
constexpr uint32_t kPBytes = kRows * 128;              // P [128 rows][64 tokens] bf16
constexpr uint32_t kMsgBytes = kPBytes + kRows * 8;    // + (rescale factor, 1 / row sum) per row
constexpr int kStage = 4;                              // score CTA: outgoing message buffers
constexpr int kRxBufs = 3;                             // output CTA: receive buffers

constexpr uint32_t kOffRingS = 0;
constexpr uint32_t kOffStage = kOffRingS + kSlotsS * kSlotBytesS;   // score CTA: outgoing messages
constexpr uint32_t kOffRx = 0;                         // output CTA: messages of the tiles in flight
constexpr uint32_t kOffRingO = kOffRx + kRxBufs * kMsgBytes;
constexpr uint32_t kEndS = kOffStage + kStage * kMsgBytes, kEndO = kOffRingO + kHalvesO * kHalf;
constexpr uint32_t kOffCtl = (kEndS > kEndO ? kEndS : kEndO);
constexpr uint32_t kSmemBytes = kOffCtl + 4096 + 1024;     // control block + alignment slack
static_assert(kSlotBytesS % 1024 == 0 && kOffRingO % 1024 == 0 && kMsgBytes % 1024 == 0 && kOffCtl % 1024 == 0,
              "swizzled buffers need 1024-byte alignment");
static_assert(kSmemBytes <= 232448, "shared memory budget");

// TMEM columns. Score CTA: the absorbed query (bf16 pairs, 288 columns = 576 channels) and one
// score buffer of 128 columns (a tile pair); output CTA: O.
constexpr uint32_t kTmemQ = 0;
constexpr uint32_t kTmemS = 288;
constexpr uint32_t kTmemCols = 512;
static_assert(kTmemS + 128 <= kTmemCols, "TMEM budget of the score CTA");

constexpr int kRowThreads = 256;   // warps 0-7: softmax (score CTA) / row work (output CTA)
constexpr int kThreads = kRowThreads + 96;
constexpr int kProducerWarp = 8;
constexpr int kMmaWarp = 9;
constexpr int kPostWarp = 10;      // score CTA: copies each written message to the output CTA
constexpr float kRescaleThreshold = 8.0f;

struct Ctl {
  // score CTA
  uint64_t full[kSlotsS], empty[kSlotsS];
  uint64_t q_full, q_empty;
  uint64_t s_full, s_empty;
  uint64_t written[kStage];     // the 128 softmax threads of a tile wrote its message into buffer s
  uint64_t sent[kStage];        // the message in buffer s reached the output CTA (s is free again)
  uint64_t credit[kRxBufs];     // the output CTA's PV that read receive buffer b has completed
  // output CTA
  uint64_t ofull[kHalvesO], oempty[kHalvesO];
  uint64_t rx_full[kRxBufs];    // the message of a tile landed in receive buffer b
  uint64_t p_ready[kRxBufs];    // rows of buffer b checked (rescaled, tail zeroed): PV may run
  uint64_t pv_done[kRxBufs];
  uint64_t drain;
  uint64_t xbar[4];          // score CTA: the two softmax warps of lane quarter q posted their maxima
  uint64_t sbar[4];          // ... their row sums (a segment's last pair)
  uint32_t tmem_base;
  int abort;
  WorkerPlan plan;
  float xmax[2][2][kRows];   // score CTA: [pair parity][column half][row] partial row maxima
  float xsum[2][kRows];      // score CTA: [column half][row] row sums at a segment's end
};
static_assert(sizeof(Ctl) <= 4096, "control block");

// One arrival for the whole warp, after every lane's earlier memory operations (the barriers
// that warps 0-7 signal count warps, not threads).
__device__ __forceinline__ void warp_arrive(uint32_t bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Physical block of tile `tile` of sequence b; an id out of range sets the status word and
// maps to the block just past the cache, which TMA reads as zeros.
__device__ __forceinline__ int tile_block(const DecodeArgs& a, int b, int tile) {
  const int blk = __ldg(a.block_table + (size_t)b * a.max_blocks + tile);
  if (blk < 0 || blk >= a.num_blocks) {
    set_status(a.status, MLA_ERR_BAD_BLOCK_ID);
    return a.num_blocks;
  }
  return blk;
}

// Prefetch into L2 the query rows of row group rg of sequence b (latent and RoPE parts), so the
// softmax warps' loads of a new segment's query hit L2: the score MMAs wait for them.
__device__ __forceinline__ void prefetch_query(const DecodeArgs& a, int b, int rg) {
  const int r0 = rg * kRows, nr = min(kRows, a.rows - r0);
  if (nr <= 0) return;
  const size_t row = (size_t)b * a.rows + r0;
  prefetch_l2((const uint16_t*)a.q_lat + row * kR, (uint32_t)nr * kR * 2);
  prefetch_l2((const uint16_t*)a.q_rope + row * kDR, (uint32_t)nr * kDR * 2);
}

// Physical cache row of entry j of sequence b's selected-token list (sparse decode). Entries
// past the count, and entries whose position or block id is out of range (which also sets the
// status word), map to the row just past the cache, which the row gathers read as zeros.
__device__ __forceinline__ int sparse_row(const DecodeArgs& a, int b, int j, int count) {
  const int oob = a.num_blocks * kBS;
  if (j >= count) return oob;
  const int t = __ldg(a.sel_idx + (size_t)b * a.top_k + j);
  const int blk = (t >= 0 && t < a.max_blocks * kBS) ? __ldg(a.block_table + (size_t)b * a.max_blocks + t / kBS) : -1;
  if (blk < 0 || blk >= a.num_blocks) {
    set_status(a.status, MLA_ERR_BAD_BLOCK_ID);
    return oob;
  }
  return blk * kBS + t % kBS;
}

// kSparse: tile t of a sequence is entries [64 t, 64 t + 64) of its selected-token list (the
// sparse decode); tm_kv is then the cache as rows [num_blocks * 64][576] (one-row boxes of 64
// channels, 128-byte swizzle) and the producers fetch each tile's rows with 4-row gathers.
template <bool kSparse>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    pair_decode_kernel(const __grid_constant__ CUtensorMap tm_kv, const __grid_constant__ CUtensorMap tm_kv4,
                       const DecodeArgs a, const int n_rg,
                       const uint64_t timeout_ns, const uint64_t drain_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  Ctl& ctl = *reinterpret_cast<Ctl*>(smem + kOffCtl);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();   // 0: scores and softmax, 1: output
  const uint32_t peer = rank ^ 1u;
  const int cluster = (int)(blockIdx.x >> 1);
  const int w = cluster / n_rg, rg = cluster % n_rg;
  const int cap = a.len_cap;
  volatile int* abort = &ctl.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSlotsS; ++i) {
      mbar_init(smem_u32(&ctl.full[i]), 1);
      mbar_init(smem_u32(&ctl.empty[i]), 1);
    }
    mbar_init(smem_u32(&ctl.q_full), kRowThreads / 32);   // one arrival per warp
    mbar_init(smem_u32(&ctl.q_empty), 1);
    mbar_init(smem_u32(&ctl.s_full), 1);
    mbar_init(smem_u32(&ctl.s_empty), kRowThreads / 32);
    for (int i = 0; i < kHalvesO; ++i) {
      mbar_init(smem_u32(&ctl.ofull[i]), 1);
      mbar_init(smem_u32(&ctl.oempty[i]), 1);
    }
    for (int i = 0; i < kStage; ++i) {
      mbar_init(smem_u32(&ctl.written[i]), 4);   // the four warps of one tile
      mbar_init(smem_u32(&ctl.sent[i]), 1);
    }
    for (int i = 0; i < kRxBufs; ++i) {
      mbar_init(smem_u32(&ctl.credit[i]), 1);
      mbar_init(smem_u32(&ctl.rx_full[i]), 1);
      // receive buffers armed for tiles 0 .. kRxBufs - 1
      if (rank == 1) mbar_arrive_expect_tx(smem_u32(&ctl.rx_full[i]), kMsgBytes);
      mbar_init(smem_u32(&ctl.p_ready[i]), kRowThreads / 32);
      mbar_init(smem_u32(&ctl.pv_done[i]), 1);
    }
    mbar_init(smem_u32(&ctl.drain), 1);
    for (int i = 0; i < 4; ++i) {
      mbar_init(smem_u32(&ctl.xbar[i]), 2);
      mbar_init(smem_u32(&ctl.sbar[i]), 2);
    }
    ctl.abort = 0;
    fence_mbarrier_init_cluster();
  }
  if (warp == kProducerWarp) {
    const WorkerPlan p = warp_plan(a.seq_lens, a.B, a.bs, cap, a.W, w, a.status);
    if (lane == 0) {
      ctl.plan = p;
      prefetch_tmap(rank == 0 ? &tm_kv : &tm_kv4);
    }
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(&ctl.tmem_base), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  cluster_sync();   // both CTAs' barriers initialised, TMEM allocated, plan ready
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;
  const WorkerPlan plan = ctl.plan;

  auto wait_warp = [&](uint32_t bar, uint32_t parity) {
    return __all_sync(0xffffffffu, mbar_wait<false>(bar, parity, abort, timeout_ns));
  };

  // Geometry of warps 0-7 (both CTAs): thread = TMEM lane = query row of the group; warp q and
  // q + 4 share the rows of lane quarter q and split the columns (half = warp / 4).
  const int quarter = warp & 3, half = (warp >> 2) & 1;
  const int row = 32 * quarter + lane;
  const uint32_t lane_off = (uint32_t)(32 * quarter) << 16;
  const int grow = rg * kRows + row;
  const bool valid_row = grow < a.rows;
  const int s_idx = valid_row ? grow / a.H : 0;

  if (kSparse && rank == 0 && warp == kProducerWarp) {
    // ------------------------------------------------------------------ score CTA: row gathers
    // lane L fetches rows 4L .. 4L + 3 of the tile pair (entries 64 tile + 4L + m), each of the
    // slot's three 64-channel chunks with one 4-row gather: the same slot layout as the tiled
    // loads (second tile's rows right after the first's).
    SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
    Segment sg;
    uint32_t c = 0;   // slots issued
    bool ok = true;
    while (ok && it.next(sg)) {
      if (lane == 0) prefetch_query(a, sg.b, rg);
      for (int tile = sg.tile_begin; ok && tile < sg.tile_end; tile += 2) {
        const int nt = min(2, sg.tile_end - tile);
        const bool act = lane < 16 * nt;
        int r4[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) r4[m] = act ? sparse_row(a, sg.b, tile * kBS + 4 * lane + m, sg.Lc) : 0;
#pragma unroll 1   // rolled: see the score MMA loop
        for (int g = 0; g < kChunksS / kGroupS; ++g, ++c) {
          const uint32_t slot = c % kSlotsS;
          bool free_slot = true;
          if (lane == 0 && c >= (uint32_t)kSlotsS)
            free_slot = mbar_wait<false>(smem_u32(&ctl.empty[slot]), ((c / kSlotsS) & 1) ^ 1, abort, timeout_ns);
          ok = __shfl_sync(0xffffffffu, free_slot, 0);
          if (!ok) break;
          const uint32_t bar = smem_u32(&ctl.full[slot]);
          const uint32_t dst = smem_u32(smem + kOffRingS + slot * kSlotBytesS);
          if (lane == 0) mbar_arrive_expect_tx(bar, nt * kGroupS * kChunk);
          __syncwarp();
          if (act) {
#pragma unroll
            for (int jj = 0; jj < kGroupS; ++jj)
              tma_gather4(dst + jj * kDChunk + lane * 512, &tm_kv, bar, 64 * (kGroupS * g + jj), r4);
          }
        }
      }
    }
    if (lane == 0) {
      int dummy = 0;
      for (uint32_t i = 0; i < kSlotsS && i < c; ++i) {
        const uint32_t cl = c - 1 - i;
        mbar_wait<false>(smem_u32(&ctl.full[cl % kSlotsS]), (cl / kSlotsS) & 1, &dummy, drain_ns);
      }
      if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
    }
  } else if (rank == 0 && warp == kProducerWarp) {
    // ------------------------------------------------------------------ score CTA: TMA producer
    if (lane == 0) {
      // (An L2 prefetch of whole blocks a few tiles ahead of these loads measured slower on
      // B200, the farther ahead the slower: the ring's own loads are the only reads.)
      SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
      Segment sg;
      uint32_t c = 0;   // slots issued
      bool ok = true;
      while (ok && it.next(sg)) {
        prefetch_query(a, sg.b, rg);
        for (int tile = sg.tile_begin; ok && tile < sg.tile_end; tile += 2) {
          const int nt = min(2, sg.tile_end - tile);
          const int blk0 = tile_block(a, sg.b, tile);
          const int blk1 = nt == 2 ? tile_block(a, sg.b, tile + 1) : 0;
#pragma unroll 1   // rolled: see the score MMA loop
          for (int g = 0; g < kChunksS / kGroupS; ++g, ++c) {
            const uint32_t slot = c % kSlotsS;
            if (c >= (uint32_t)kSlotsS &&
                !mbar_wait<false>(smem_u32(&ctl.empty[slot]), ((c / kSlotsS) & 1) ^ 1, abort, timeout_ns)) {
              ok = false;
              break;
            }
            const uint32_t bar = smem_u32(&ctl.full[slot]);
            const uint32_t dst = smem_u32(smem + kOffRingS + slot * kSlotBytesS);
            mbar_arrive_expect_tx(bar, nt * kGroupS * kChunk);
            // chunk j of the pair's first tile, then of the second, for kGroupS consecutive chunks
#pragma unroll
            for (int jj = 0; jj < kGroupS; ++jj) {
              const int j = kGroupS * g + jj;
              tma_load_3d(dst + jj * kDChunk, &tm_kv, bar, 64 * j, 0, blk0);
              if (nt == 2) tma_load_3d(dst + jj * kDChunk + kChunk, &tm_kv, bar, 64 * j, 0, blk1);
            }
          }
        }
      }
      // every load issued has landed before the CTA may exit
      int dummy = 0;
      for (uint32_t i = 0; i < kSlotsS && i < c; ++i) {
        const uint32_t cl = c - 1 - i;
        mbar_wait<false>(smem_u32(&ctl.full[cl % kSlotsS]), (cl / kSlotsS) & 1, &dummy, drain_ns);
      }
      if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
    }
  } else if (rank == 0 && warp == kMmaWarp) {
    // ------------------------------------------------------------------ score CTA: MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc2 = idesc_bf16_f32(128, 128, false);   // a tile pair
      constexpr uint32_t idesc1 = idesc_bf16_f32(128, 64, false);    // a single tile
      SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
      Segment sg;
      uint32_t c = 0, u = 0, seg = 0;
      bool ok = true;
      while (ok && it.next(sg)) {
        ok = mbar_wait<false>(smem_u32(&ctl.q_full), seg & 1, abort, timeout_ns);
        if (!ok) break;
        tc_fence_after();
        for (int tile = sg.tile_begin; ok && tile < sg.tile_end; tile += 2, ++u) {
          const uint32_t idesc = sg.tile_end - tile >= 2 ? idesc2 : idesc1;
          if (u >= 1) ok = mbar_wait<false>(smem_u32(&ctl.s_empty), (u & 1) ^ 1, abort, timeout_ns);
          if (!ok) break;
          tc_fence_after();
          // Loops around barrier waits stay rolled: unrolled, the pipelines of this kernel ran about
          // 1.4x slower on B200 (measured).
#pragma unroll 1
          for (int g = 0; g < kChunksS / kGroupS; ++g, ++c) {
            const uint32_t slot = c % kSlotsS;
            ok = mbar_wait<false>(smem_u32(&ctl.full[slot]), (c / kSlotsS) & 1, abort, timeout_ns);
            if (!ok) break;
            tc_fence_after();
            const uint32_t base = smem_u32(smem + kOffRingS + slot * kSlotBytesS);
#pragma unroll
            for (int jj = 0; jj < kGroupS; ++jj) {
              const int j = kGroupS * g + jj;
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) {
                // channels [64 j + 16 kk, +16): A = query words from TMEM, B = the pair's rows of
                // chunk j (K-major, 8-row groups 1 KB apart, the second tile right after the first)
                const uint64_t bdesc = smem_desc(base + jj * kDChunk + kk * 32, 16, 1024, kSwizzle128B);
                mma_ts(tmem + kTmemS, tmem + kTmemQ + 8 * (4 * j + kk), bdesc, idesc, (j | kk) ? 1u : 0u);
              }
            }
            mma_commit(smem_u32(&ctl.empty[slot]));   // the slot is free once these MMAs have read it
          }
          if (!ok) break;
          mma_commit(smem_u32(&ctl.s_full));
        }
        if (!ok) break;
        mma_commit(smem_u32(&ctl.q_empty));
        ++seg;
      }
      int dummy = 0;
      mma_commit(smem_u32(&ctl.drain));
      mbar_wait<false>(smem_u32(&ctl.drain), 0, &dummy, drain_ns);
      if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
    }
  } else if (rank == 0 && warp < kProducerWarp) {
    // ------------------------------------------------------------------ score CTA: softmax warps
    const float scale_log2 = a.scale_log2;
    SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
    Segment sg;
    uint32_t t = 0, u = 0, seg = 0;   // tiles and pairs before this segment, segments
    bool ok = true;
    while (it.next(sg)) {
      const int n = sg.tile_end - sg.tile_begin;
      float m_run = -INFINITY, l_run = 0.f, l_tot = 0.f;   // l_run: this half's columns
      if (ok) {
        // this segment's absorbed query into TMEM, one row per thread pair: half 0 loads the
        // latent channels [0, 256), half 1 the channels [256, 512) and the RoPE channels
        ok = wait_warp(smem_u32(&ctl.q_empty), (seg & 1) ^ 1);
        if (ok) {
          const size_t qoff = (size_t)sg.b * a.rows + (valid_row ? grow : 0);
          const uint4* ql = reinterpret_cast<const uint4*>((const uint16_t*)a.q_lat + qoff * kR) + 32 * half;
          const uint4* qr = reinterpret_cast<const uint4*>((const uint16_t*)a.q_rope + qoff * kDR);
          const int nq = half ? 40 : 32;   // 16-byte pieces of this thread's share (multiples of 8)
#pragma unroll 1
          for (int r0 = 0; r0 < nq; r0 += 16) {
            uint4 qv[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const int k = r0 + i;
              qv[i] = (valid_row && k < nq) ? __ldg(k < 32 ? ql + k : qr + (k - 32)) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int g = 0; g < 16; g += 8) {
              const int k = r0 + g;   // first piece of this group of 8 (32 columns)
              if (k < nq) {
                uint32_t w32[32];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                  w32[4 * i] = qv[g + i].x;
                  w32[4 * i + 1] = qv[g + i].y;
                  w32[4 * i + 2] = qv[g + i].z;
                  w32[4 * i + 3] = qv[g + i].w;
                }
                // piece k holds query words 4 k .. 4 k + 3 of this half's latent block, or (k >= 32)
                // the RoPE words 4 (k - 32) .. ; column = word index
                const uint32_t col = k < 32 ? 128 * half + 4 * k : 256 + 4 * (k - 32);
                tmem_st32(tmem + lane_off + kTmemQ + col, w32);
              }
            }
          }
          tmem_wait_st();
          tc_fence_before();
          warp_arrive(smem_u32(&ctl.q_full));
        }
        int n_row = valid_row ? (a.causal ? sg.Lc - a.Sq + 1 + s_idx : sg.Lc) : 0;
        if (n_row < 0) n_row = 0;
        for (int li = 0; ok && li < n; li += 2, ++u) {
          const int nt = min(2, n - li);            // tiles in this pair
          const bool mine = half < nt;              // this half has a tile
          const int tile = sg.tile_begin + li + half;
          const bool last_pair = li + 2 >= n;
          ok = wait_warp(smem_u32(&ctl.s_full), u & 1);
          if (!ok) break;
          tc_fence_after();
          uint32_t v[64];
          tmem_ld32(tmem + lane_off + kTmemS + 64 * half, v);
          tmem_ld32(tmem + lane_off + kTmemS + 64 * half + 32, v + 32);
          tmem_wait_ld();
          tc_fence_before();
          warp_arrive(smem_u32(&ctl.s_empty));
          // The pair's row maximum of the scaled scores (log2 units) from both halves. A full tile
          // keeps the raw scores and takes the extreme with three-input min / max (the scale folds
          // into the exponent's FMA below); a partial one masks the columns past the row's
          // attended tokens after scaling.
          const int valid = mine ? min(max(n_row - tile * kBS, 0), kBS) : 0;
          const bool full = valid == kBS;
          float mh;
          if (full) {
            float r = __uint_as_float(v[0]);
            if (scale_log2 >= 0.f) {
#pragma unroll
              for (int j = 1; j < 63; j += 2) r = max3f(r, __uint_as_float(v[j]), __uint_as_float(v[j + 1]));
              r = fmaxf(r, __uint_as_float(v[63]));
            } else {
#pragma unroll
              for (int j = 1; j < 63; j += 2) r = min3f(r, __uint_as_float(v[j]), __uint_as_float(v[j + 1]));
              r = fminf(r, __uint_as_float(v[63]));
            }
            mh = r * scale_log2;
          } else {
            mh = -INFINITY;
#pragma unroll
            for (int j = 0; j < 64; ++j) {
              const float x = j < valid ? __uint_as_float(v[j]) * scale_log2 : -INFINITY;
              v[j] = __float_as_uint(x);
              mh = fmaxf(mh, x);
            }
          }
          ctl.xmax[u & 1][half][row] = mh;
          warp_arrive(smem_u32(&ctl.xbar[quarter]));
          ok = wait_warp(smem_u32(&ctl.xbar[quarter]), u & 1);   // bounded: the partner warp may have aborted
          if (!ok) break;
          const float mt = fmaxf(mh, ctl.xmax[u & 1][half ^ 1][row]);
          const bool grow_max = mt > m_run + kRescaleThreshold;
          const float alpha = (grow_max && m_run != -INFINITY) ? ex2_approx(m_run - mt) : 1.f;
          if (grow_max) {
            l_run *= alpha;
            m_run = mt;
          }
          uint32_t pk[32];
          float psum = 0.f;
          if (m_run != -INFINITY) {
            // p = 2^(c s - m) two columns at a time: c = the scale (full tile) or 1 (scaled, masked)
            const float c = full ? scale_log2 : 1.f;
            const unsigned long long cc = f2_pack(c, c), nm = f2_pack(-m_run, -m_run);
            unsigned long long acc = f2_pack(0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 32; ++k) {
              float x0, x1;
              f2_unpack(fma2(f2_pack(__uint_as_float(v[2 * k]), __uint_as_float(v[2 * k + 1])), cc, nm), x0, x1);
              const float p0 = ex2_approx(x0), p1 = ex2_approx(x1);
              acc = add2(acc, f2_pack(p0, p1));
              pk[k] = pack_bf16x2(p0, p1);
            }
            float s0, s1;
            f2_unpack(acc, s0, s1);
            psum = s0 + s1;
          } else {
#pragma unroll
            for (int k = 0; k < 32; ++k) pk[k] = 0u;
          }
          l_run += psum;
          if (last_pair) {
            // the segment's row sum over both halves, for the output CTA's normalisation
            ctl.xsum[half][row] = l_run;
            warp_arrive(smem_u32(&ctl.sbar[quarter]));
            ok = wait_warp(smem_u32(&ctl.sbar[quarter]), seg & 1);
            if (!ok) break;
            l_tot = l_run + ctl.xsum[half ^ 1][row];
          }
          if (mine) {
            const bool last_tile = last_pair && half == nt - 1;
            const float invl = (last_tile && l_tot > 0.f) ? 1.f / l_tot : 0.f;
            // O is rescaled before the pair's first tile only
            const float fac = half == 0 ? alpha : 1.f;
            // outgoing buffer tt % kStage is free once tile tt - kStage has reached the output CTA
            const uint32_t tt = t + li + half, sb = tt % kStage;
            bool free_buf = true;
            if (lane == 0 && tt >= (uint32_t)kStage)
              free_buf = mbar_wait<true>(smem_u32(&ctl.sent[sb]), ((tt / kStage) & 1) ^ 1, abort, timeout_ns);
            ok = __shfl_sync(0xffffffffu, free_buf, 0);
            if (!ok) break;
            // this row of the tile's message: P as [8-token chunk][row][8 tokens] (8-row x 16-byte
            // core matrices, the K-major layout the output CTA's PV reads), then the row's
            // (rescale factor, 1 / row sum)
            uint8_t* msg = smem + kOffStage + sb * kMsgBytes;
#pragma unroll
            for (int cc = 0; cc < 8; ++cc)
              *reinterpret_cast<uint4*>(msg + cc * (kRows * 16) + row * 16) =
                  make_uint4(pk[4 * cc], pk[4 * cc + 1], pk[4 * cc + 2], pk[4 * cc + 3]);
            *reinterpret_cast<float2*>(msg + kPBytes + row * 8) = make_float2(fac, invl);
            fence_proxy_async_smem();   // for the bulk copy that sends the buffer
            warp_arrive(smem_u32(&ctl.written[sb]));
          }
        }
        t += n;
        ++seg;
      }
      // log-sum-exp of the rows of this segment (the output CTA writes the values)
      const bool poisoned = segment_poisoned(a, sg.b, sg.tile_begin, sg.tile_end);
      if (valid_row && half == 0) {
        float lse_v = l_tot > 0.f ? (m_run + log2f(l_tot)) * 0.69314718055994531f : -INFINITY;
        if (!ok || poisoned) lse_v = __uint_as_float(0x7FC00000u);
        if (sg.splits == 1)
          a.lse[(size_t)sg.b * a.rows + grow] = lse_v;
        else
          a.lse_part[(size_t)(w + sg.b) * a.rows + grow] = lse_v;
      }
    }
    if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
  } else if (rank == 0 && warp == kPostWarp) {
    // ------------------------------------------------------------------ score CTA: message sends
    // In tile order: once the 128 softmax threads of a tile have written its message and the
    // PV that last read receive buffer t % kRxBufs has completed, one bulk copy moves the
    // message into the output CTA's shared memory (bytes complete on its barrier).
    if (lane == 0) {
      SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
      Segment sg;
      uint32_t t = 0;
      bool ok = true;
      while (ok && it.next(sg)) {
        for (int li = sg.tile_begin; li < sg.tile_end; ++li, ++t) {
          const uint32_t sb = t % kStage, rb = t % kRxBufs;
          ok = mbar_wait<false>(smem_u32(&ctl.written[sb]), (t / kStage) & 1, abort, timeout_ns);
          if (ok && t >= (uint32_t)kRxBufs)
            ok = mbar_wait<true>(smem_u32(&ctl.credit[rb]), ((t / kRxBufs) & 1) ^ 1, abort, timeout_ns);
          if (!ok) break;
          bulk_copy_to_peer(mapa(smem_u32(smem + kOffRx + rb * kMsgBytes), peer),
                            smem_u32(smem + kOffStage + sb * kMsgBytes), kMsgBytes,
                            mapa(smem_u32(&ctl.rx_full[rb]), peer));
        }
      }
      // the PV completions of the last tiles still signal our credit barriers: wait for them
      // (bounded) so that no arrival can reach this CTA's shared memory after it exits
      int dummy = 0;
      for (uint32_t i = 0; i < (uint32_t)kRxBufs && i < t; ++i) {
        const uint32_t tl = t - 1 - i;
        mbar_wait<true>(smem_u32(&ctl.credit[tl % kRxBufs]), (tl / kRxBufs) & 1, &dummy, drain_ns);
      }
      if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
    }
  } else if (kSparse && warp == kProducerWarp) {
    // ------------------------------------------------------------------ output CTA: row gathers
    // lanes 0-15 fetch the tile's rows 4L .. 4L + 3, each half stage's four 64-channel chunks
    // with one 4-row gather each (the layout of the tiled 4-D box)
    SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
    Segment sg;
    uint32_t h = 0;
    bool ok = true;
    while (ok && it.next(sg)) {
      for (int tile = sg.tile_begin; ok && tile < sg.tile_end; ++tile) {
        const bool act = lane < 16;
        int r4[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) r4[m] = act ? sparse_row(a, sg.b, tile * kBS + 4 * lane + m, sg.Lc) : 0;
#pragma unroll 1   // rolled: see the score MMA loop
        for (int hc = 0; hc < 2; ++hc, ++h) {
          const uint32_t hs = h % kHalvesO;
          bool free_half = true;
          if (lane == 0 && h >= (uint32_t)kHalvesO)
            free_half = mbar_wait<false>(smem_u32(&ctl.oempty[hs]), ((h / kHalvesO) & 1) ^ 1, abort, timeout_ns);
          ok = __shfl_sync(0xffffffffu, free_half, 0);
          if (!ok) break;
          const uint32_t bar = smem_u32(&ctl.ofull[hs]);
          const uint32_t base = smem_u32(smem + kOffRingO + hs * kHalf);
          if (lane == 0) mbar_arrive_expect_tx(bar, kHalf);
          __syncwarp();
          if (act) {
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
              tma_gather4(base + cc * kChunk + lane * 512, &tm_kv, bar, 256 * hc + 64 * cc, r4);
          }
        }
      }
    }
    if (lane == 0) {
      int dummy = 0;
      for (uint32_t i = 0; i < kHalvesO && i < h; ++i) {
        const uint32_t hl = h - 1 - i;
        mbar_wait<false>(smem_u32(&ctl.ofull[hl % kHalvesO]), (hl / kHalvesO) & 1, &dummy, drain_ns);
      }
      if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
    }
  } else if (warp == kProducerWarp) {
    // ------------------------------------------------------------------ output CTA: TMA producer
    if (lane == 0) {
      SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
      Segment sg;
      uint32_t h = 0;
      bool ok = true;
      while (ok && it.next(sg)) {
        for (int tile = sg.tile_begin; ok && tile < sg.tile_end; ++tile) {
          const int blk = tile_block(a, sg.b, tile);
#pragma unroll 1   // rolled: see the score MMA loop
          for (int hc = 0; hc < 2; ++hc, ++h) {
            const uint32_t hs = h % kHalvesO;
            if (h >= (uint32_t)kHalvesO &&
                !mbar_wait<false>(smem_u32(&ctl.oempty[hs]), ((h / kHalvesO) & 1) ^ 1, abort, timeout_ns)) {
              ok = false;
              break;
            }
            const uint32_t bar = smem_u32(&ctl.ofull[hs]);
            const uint32_t base = smem_u32(smem + kOffRingO + hs * kHalf);
            mbar_arrive_expect_tx(bar, kHalf);
            tma_load_4d(base, &tm_kv4, bar, 0, 0, 4 * hc, blk);   // latent chunks 4 hc .. 4 hc + 3
          }
        }
      }
      int dummy = 0;
      for (uint32_t i = 0; i < kHalvesO && i < h; ++i) {
        const uint32_t hl = h - 1 - i;
        mbar_wait<false>(smem_u32(&ctl.ofull[hl % kHalvesO]), (hl / kHalvesO) & 1, &dummy, drain_ns);
      }
      if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
    }
  } else if (warp == kMmaWarp) {
    // ------------------------------------------------------------------ output CTA: MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, 256, true);
      const uint32_t rx = smem_u32(smem + kOffRx);
      SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
      Segment sg;
      uint32_t t = 0, h = 0;
      bool ok = true;
      while (ok && it.next(sg)) {
        const int n = sg.tile_end - sg.tile_begin;
        for (int li = 0; li < n; ++li, ++t) {
          const uint32_t rb = t % kRxBufs;
          ok = mbar_wait<false>(smem_u32(&ctl.p_ready[rb]), (t / kRxBufs) & 1, abort, timeout_ns);
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1   // rolled: see the score MMA loop
          for (int hc = 0; hc < 2; ++hc, ++h) {
            const uint32_t hs = h % kHalvesO;
            ok = mbar_wait<false>(smem_u32(&ctl.ofull[hs]), (h / kHalvesO) & 1, abort, timeout_ns);
            if (!ok) break;
            tc_fence_after();
            const uint32_t base = smem_u32(smem + kOffRingO + hs * kHalf);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              // A = P[128 rows][tokens 16 kk .. +16] (K-major); B = C[16 tokens][256 channels],
              // channels contiguous: 64-channel chunks 8 KB apart, 8-token groups 1 KB apart
              // (the message's P: 8-row x 16-byte core matrices, 128 bytes apart along the rows,
              // 2 KB apart along the tokens)
              const uint64_t adesc = smem_desc(rx + rb * kMsgBytes + kk * 4096, 2048, 128, kSwizzleNone);
              const uint64_t bdesc = smem_desc(base + kk * 2048, kChunk, 1024, kSwizzle128B);
              mma_ss(tmem + 256 * hc, adesc, bdesc, idesc_pv, (li > 0 || kk > 0) ? 1u : 0u);
            }
            mma_commit(smem_u32(&ctl.oempty[hs]));
          }
          if (!ok) break;
          mma_commit(smem_u32(&ctl.pv_done[rb]));   // O is free again after this PV
          // the receive buffer goes back to the score CTA when this PV has completed
          mma_commit_to_ctas(smem_u32(&ctl.credit[rb]), (uint16_t)(1u << peer));
        }
      }
      int dummy = 0;
      mma_commit(smem_u32(&ctl.drain));
      mbar_wait<false>(smem_u32(&ctl.drain), 0, &dummy, drain_ns);
      if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
    }
  } else if (warp < kProducerWarp) {
    // ------------------------------------------------------------------ output CTA: row warps
    // thread = row; warp q works on O columns [0, 256) of its rows, warp q + 4 on [256, 512)
    const uint32_t rx = smem_u32(smem + kOffRx);
    const uint32_t col0 = 256 * half;
    SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
    Segment sg;
    uint32_t t = 0;
    bool ok = true;
    while (it.next(sg)) {
      const int n = sg.tile_end - sg.tile_begin;
      float inv_l = 0.f;
      if (ok) {
        const int last_tile = (sg.Lc + kBS - 1) / kBS - 1;
        const int tail = sg.Lc % kBS;
        for (int li = 0; li < n; ++li, ++t) {
          const uint32_t rb = t % kRxBufs, sb = t % kStage;
          const int tile = sg.tile_begin + li;
          ok = wait_warp(smem_u32(&ctl.rx_full[rb]), (t / kRxBufs) & 1);
          if (!ok) break;
          if (threadIdx.x == 0) {
            // re-arm for tile t + kRxBufs (its bytes can only come after this tile's PV), and hand
            // the score CTA's outgoing buffer of this tile back (the copy has read it)
            mbar_arrive_expect_tx(smem_u32(&ctl.rx_full[rb]), kMsgBytes);
            mbar_arrive_remote_relaxed(mapa(smem_u32(&ctl.sent[sb]), peer));
          }
          float2 fl;
          asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];"
                       : "=f"(fl.x), "=f"(fl.y)
                       : "r"(rx + rb * kMsgBytes + kPBytes + (uint32_t)row * 8));
          const float alpha = fl.x;
          if (li == n - 1) inv_l = fl.y;
          if (li >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
            // O holds the tiles before t: wait for their PV, then scale this row's half
            const uint32_t tp = t - 1;
            ok = wait_warp(smem_u32(&ctl.pv_done[tp % kRxBufs]), (tp / kRxBufs) & 1);
            if (!ok) break;
            tc_fence_after();
#pragma unroll 1
            for (int cc = 0; cc < 8; ++cc) {
              uint32_t v[32];
              tmem_ld32(tmem + lane_off + col0 + 32 * cc, v);
              tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = __float_as_uint(__uint_as_float(v[i]) * alpha);
              tmem_st32(tmem + lane_off + col0 + 32 * cc, v);
            }
            tmem_wait_st();
          }
          if (tile == last_tile && tail != 0) {
            // cache slots past the sequence end may hold anything (NaN): zero those token rows
            // of both half stages before the PV reads them (P is 0 there, but 0 * NaN is not)
            const uint32_t h0 = 2 * t, h1 = 2 * t + 1;
            ok = wait_warp(smem_u32(&ctl.ofull[h0 % kHalvesO]), (h0 / kHalvesO) & 1) &&
                 wait_warp(smem_u32(&ctl.ofull[h1 % kHalvesO]), (h1 / kHalvesO) & 1);
            if (!ok) break;
            const int per_chunk = (kBS - tail) * 8;   // 16-byte pieces per chunk
            for (int i = threadIdx.x; i < 8 * per_chunk; i += kRowThreads) {
              const int ck = i / per_chunk, rem = i % per_chunk;
              const uint32_t hs = (ck < 4 ? h0 : h1) % kHalvesO;
              uint8_t* p = smem + kOffRingO + hs * kHalf + (ck & 3) * kChunk + (tail + rem / 8) * 128 + (rem % 8) * 16;
              *reinterpret_cast<uint4*>(p) = make_uint4(0u, 0u, 0u, 0u);
            }
            fence_proxy_async_smem();
          }
          tc_fence_before();
          warp_arrive(smem_u32(&ctl.p_ready[rb]));
        }
        if (ok) ok = wait_warp(smem_u32(&ctl.pv_done[(t - 1) % kRxBufs]), ((t - 1) / kRxBufs) & 1);
      }
      // epilogue: O / l -> out (single split) or the normalised partial (several splits)
      const bool poisoned = segment_poisoned(a, sg.b, sg.tile_begin, sg.tile_end);
      const bool nan_rows = !ok || poisoned;
      const bool direct = sg.splits == 1;
      const size_t qrow = (size_t)sg.b * a.rows + grow;
      const size_t prow = (size_t)(w + sg.b) * a.rows + grow;
      if (ok) tc_fence_after();
#pragma unroll 1
      for (int cc = 0; cc < 8; ++cc) {
        uint32_t v[32];
        if (ok) {
          tmem_ld32(tmem + lane_off + col0 + 32 * cc, v);
          tmem_wait_ld();
        }
        if (!valid_row) continue;
        float f[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) f[i] = nan_rows ? __uint_as_float(0x7FC00000u) : __uint_as_float(v[i]) * inv_l;
        const int ch = col0 + 32 * cc;
        if (direct && a.out_dtype == kBF16) {
          uint4* dst = reinterpret_cast<uint4*>((uint16_t*)a.out + qrow * kR + ch);
#pragma unroll
          for (int i = 0; i < 4; ++i)
            dst[i] = make_uint4(pack_bf16x2(f[8 * i], f[8 * i + 1]), pack_bf16x2(f[8 * i + 2], f[8 * i + 3]),
                                pack_bf16x2(f[8 * i + 4], f[8 * i + 5]), pack_bf16x2(f[8 * i + 6], f[8 * i + 7]));
        } else {
          float4* dst = reinterpret_cast<float4*>(direct ? (float*)a.out + qrow * kR + ch : a.o_part + prow * kR + ch);
#pragma unroll
          for (int i = 0; i < 8; ++i) dst[i] = make_float4(f[4 * i], f[4 * i + 1], f[4 * i + 2], f[4 * i + 3]);
        }
      }
      tc_fence_before();
    }
    if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
  }

  // ------------------------------------------------------------------ teardown
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  cluster_sync();   // no CTA leaves while its peer may still write its shared memory
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

}  // namespace

cudaError_t launch_pair_decode(const DecodeArgs& a, cudaStream_t s) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return cudaErrorInvalidValue;
  const bool sparse = a.sel_idx != nullptr;
  if (sparse && (a.Sq != 1 || a.causal)) return cudaErrorInvalidValue;
  CUtensorMap tm, tm4;
  if (sparse) {
    // the cache as rows [num_blocks * 64][576] bf16: one-row boxes of 64 channels (128 bytes,
    // 128-byte swizzle) for 4-row gathers; rows past the cache read as zeros
    const cuuint64_t dims[2] = {(cuuint64_t)(kR + kDR), (cuuint64_t)a.num_blocks * kBS};
    const cuuint64_t strides[1] = {(cuuint64_t)(kR + kDR) * 2};
    const cuuint32_t box[2] = {64, 1};
    const cuuint32_t estr[2] = {1, 1};
    if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(a.cache), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    tm4 = tm;   // unused by the gathering producers
  } else {
    // the cache [num_blocks][64][576] bf16, boxes of 64 channels x 64 tokens, 128-byte swizzle
    const cuuint64_t dims[3] = {(cuuint64_t)(kR + kDR), (cuuint64_t)kBS, (cuuint64_t)a.num_blocks};
    const cuuint64_t strides[2] = {(cuuint64_t)(kR + kDR) * 2, (cuuint64_t)kBS * (kR + kDR) * 2};
    const cuuint32_t box[3] = {64, (cuuint32_t)kBS, 1};
    const cuuint32_t estr[3] = {1, 1, 1};
    if (fn(&tm, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(a.cache), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
    // the same cache as (64 channels, 64 tokens, 9 channel chunks, blocks): one box = 4 chunks of
    // a block, written as [chunk][token][128 bytes], the layout of four 3-D boxes side by side
    const cuuint64_t dims4[4] = {64, (cuuint64_t)kBS, (cuuint64_t)(kR + kDR) / 64, (cuuint64_t)a.num_blocks};
    const cuuint64_t strides4[3] = {(cuuint64_t)(kR + kDR) * 2, 128, (cuuint64_t)kBS * (kR + kDR) * 2};
    const cuuint32_t box4[4] = {64, (cuuint32_t)kBS, 4, 1};
    const cuuint32_t estr4[4] = {1, 1, 1, 1};
    if (fn(&tm4, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(a.cache), dims4, strides4, box4, estr4,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  static std::once_flag attr_once[2][64];
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t attr_err = cudaSuccess;
  std::call_once(attr_once[sparse ? 1 : 0][dev & 63], [&] {
    attr_err = sparse ? cudaFuncSetAttribute(pair_decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemBytes)
                      : cudaFuncSetAttribute(pair_decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             kSmemBytes);
  });
  if (attr_err != cudaSuccess) return attr_err;
  const int n_rg = (a.rows + kRows - 1) / kRows;
  const dim3 grid(2 * a.W * n_rg);
  if (sparse)
    pair_decode_kernel<true><<<grid, kThreads, kSmemBytes, s>>>(tm, tm4, a, n_rg, wait_timeout_ns(), drain_timeout_ns());
  else
    pair_decode_kernel<false><<<grid, kThreads, kSmemBytes, s>>>(tm, tm4, a, n_rg, wait_timeout_ns(),
                                                                 drain_timeout_ns());
  return cudaGetLastError();
}

}  // namespace mla
