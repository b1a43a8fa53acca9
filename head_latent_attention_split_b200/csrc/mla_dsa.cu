// DeepSeek Sparse Attention side kernels ("TransMLA & Sparse Latent Attention" lesson,
// Chapter 6 "The lightning indexer" and "Fine-grained token selection"; Chapter 7 "Why
// FP8 specifically" and "The indexer keeps its own small cache").
//
// Indexer: I_t = sum_j w_j * ReLU(q_j . k_t) for every token t a query row may see, with
// H^I = 64 heads of width d^I = 128 stored as e4m3 codes with one fp32 scale per vector
// (q per head, k per cached token). Persistent CTAs (two per SM) walk contiguous ranges of
// (query row, 128-token tile) items. TMA brings each tile's key codes (two cache blocks,
// 128-byte swizzled) and key scales through a stage ring and the row's 64 x 128 query codes; one
// thread issues tcgen05 MMAs of kind::f8f6f4 with the tokens as M = 128 and the heads as
// N = 64 (K = 4 x 32 codes) into a ring of TMEM accumulators, so every TMEM lane holds one
// token's 64 head dots and the thread reading it finishes that token alone: scale, ReLU,
// weighted sum, one coalesced fp32 store. The e4m3 products are exact and summed in fp32
// by the tensor core.
//
// Top-k: a cluster of 8 CTAs (1024 threads each) per query row, each CTA on one slice of
// the row. A three-pass radix select (11, 11, 10 bits of an order-preserving key of the fp32
// score; slice histograms summed over the cluster in distributed shared memory) finds the
// k-th largest key T and how many entries equal to T are kept; an ordered pass then writes
// the positions of every score above T and of the first such ties, in ascending position
// order (block-wide scans of packed counts, offset by the lower slices' counts). Ties at T
// go to the lower positions, so the result is unique.
#include <cuda.h>

#include <algorithm>
#include <mutex>

#include "mla_device.cuh"
#include "ptx_sm100.cuh"

namespace mla {
namespace {

using namespace ptx;

// ------------------------------------------------------------------------------ indexer
// Persistent: two CTAs per SM, each walking a contiguous range of (query row, 128-token tile)
// items. Warp 4 produces (TMA: the tile's two cache blocks and their key scales into a 5-stage
// ring, the row's query into one of two slots when the row changes), warp 5 allocates TMEM
// and issues the MMAs into a ring of four 64-column accumulators, and warps 0-3 finish the
// tokens (thread = token). The per-tile handoff is latency-bound, so two independent CTAs per
// SM keep twice the tiles in flight (a second epilogue group in one CTA, kIGroups = 2, does not).
constexpr int kITok = 128;                        // tokens per tile = MMA M
constexpr int kIBlk = 64;                         // tokens per cache block
constexpr int kIStages = 5;                // TMA ring depth
constexpr int kIGroups = 1;                // epilogue warp groups (items alternate between them when 2)
constexpr int kICtasPerSm = 2;             // two independent pipelines per SM (TMEM: 2 x 256 columns)
constexpr int kIAcc = 4;
constexpr int kIThreads = 192 + 128 * (kIGroups - 1);
constexpr int kIProducer = 4, kIMma = 5;   // epilogue groups: warps 0-3 (even items), 6-9 (odd items)
constexpr uint32_t kIKTile = kITok * kDsaDim;     // 16 KB of key codes
constexpr uint32_t kIQ = kDsaHeads * kDsaDim;     // 8 KB of query codes
constexpr uint32_t kIScales = kITok * 4;          // the tile's 128 key scales (two blocks of 64)
constexpr uint32_t kITmemCols = kIAcc * kDsaHeads;

struct IdxCtl {
  uint64_t full[kIStages], empty[kIStages];
  uint64_t acc_full[kIAcc], acc_empty[kIAcc];
  uint64_t q_full[2], q_empty[2];
  uint32_t tmem_base;
  int abort;
  int r0, j0, count;   // this CTA's first item (row, tile) and its number of items
  uint32_t valid[kIStages];             // per stage: bit h set = block h of the tile was loaded
  float wq[2][kDsaHeads];               // per query slot: weight x query scale of each head
};
constexpr uint32_t kIOffQ = kIStages * kIKTile;                 // two query slots
constexpr uint32_t kIOffS = kIOffQ + 2 * kIQ;                    // key scales ring
constexpr uint32_t kIOffCtl = kIOffS + kIStages * kIScales;
static_assert(kIOffQ % 1024 == 0, "query slots need 1024-byte alignment");
constexpr uint32_t kISmem = kIOffCtl + 2048 + 1024;   // + control + alignment
static_assert(sizeof(IdxCtl) <= 2048 && kICtasPerSm * (kISmem + 1024) <= 232448, "indexer shared memory");
static_assert(kICtasPerSm * kIAcc * kDsaHeads <= 512, "TMEM columns per SM");

// tokens query row r sees; a bad seq_len flags the status and counts as 0
__device__ __forceinline__ int row_tokens(const DsaArgs& a, int r, bool report) {
  const int b = r / a.Sq, s = r % a.Sq;
  const int L = __ldg(a.seq_lens + b);
  if (L < 0 || L > a.max_blocks * a.bs || L > a.max_seq_len) {
    if (report) set_status(a.status, MLA_ERR_BAD_SEQ_LEN);
    return 0;
  }
  return max(a.causal ? L - a.Sq + 1 + s : L, 0);
}

__device__ __forceinline__ int row_tiles(const DsaArgs& a, int r) { return (row_tokens(a, r, false) + kITok - 1) / kITok; }

// walks items (row r, tile j) in order, skipping rows without tiles
struct ItemWalk {
  int r, j, T;
  __device__ void start(const DsaArgs& a, int r0, int j0) {
    r = r0;
    j = j0;
    T = r < a.B * a.Sq ? row_tiles(a, r) : 0;
  }
  __device__ void next(const DsaArgs& a) {
    if (++j >= T) {
      j = 0;
      do {
        ++r;
        T = r < a.B * a.Sq ? row_tiles(a, r) : 0;
      } while (T == 0 && r < a.B * a.Sq);
    }
  }
};

__global__ void __launch_bounds__(kIThreads, kICtasPerSm)
    dsa_index_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_s, const DsaArgs a, const uint64_t timeout_ns,
                     const uint64_t drain_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  IdxCtl& ctl = *reinterpret_cast<IdxCtl*>(smem + kIOffCtl);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int R = a.B * a.Sq;
  const uint32_t sK = smem_u32(smem), sS = smem_u32(smem + kIOffS), sQ = smem_u32(smem + kIOffQ);
  const float* scale_ring = reinterpret_cast<const float*>(smem + kIOffS);
  volatile int* abort = &ctl.abort;

  if (warp == kIProducer) {
    // this CTA's item range: [c T / G, (c + 1) T / G) of the T items of all rows
    long long T = 0;
    for (int r0 = 0; r0 < R; r0 += 32) {
      const int r = r0 + lane;
      int t = 0;
      if (r < R) t = (row_tokens(a, r, blockIdx.x == 0) + kITok - 1) / kITok;
      for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
      T += t;
    }
    const long long i0 = T * blockIdx.x / gridDim.x, i1 = T * (blockIdx.x + 1) / gridDim.x;
    if (lane == 0) {
      long long acc = 0;
      int r = 0;
      while (r < R) {
        const int t = row_tiles(a, r);
        if (acc + t > i0) break;
        acc += t;
        ++r;
      }
      ctl.r0 = r;
      ctl.j0 = (int)(i0 - acc);
      ctl.count = (int)(i1 - i0);
    }
  }
  if (threadIdx.x == 0) {
    for (int i = 0; i < kIStages; ++i) {
      mbar_init(smem_u32(&ctl.full[i]), 1);
      mbar_init(smem_u32(&ctl.empty[i]), 1 + 4);   // the tile's MMAs and each warp of its epilogue group
    }
    for (int i = 0; i < kIAcc; ++i) {
      mbar_init(smem_u32(&ctl.acc_full[i]), 1);
      mbar_init(smem_u32(&ctl.acc_empty[i]), 4);   // one arrival per warp of the item's epilogue group
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&ctl.q_full[i]), 1);
      mbar_init(smem_u32(&ctl.q_empty[i]), 1 + 4 * kIGroups);   // the MMAs of the row and each epilogue warp
    }
    ctl.abort = 0;
    fence_mbarrier_init_cluster();
  }
  if (warp == kIMma) {
    tmem_alloc(smem_u32(&ctl.tmem_base), kITmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;
  const int count = ctl.count;

  if (warp == kIProducer) {
    // ---------------------------------------------------------------- producer
    ItemWalk it;
    it.start(a, ctl.r0, ctl.j0);
    int cur_row = -1, rs = -1;   // row of the last query load, its index among this CTA's rows
    int issued = 0;              // items whose loads are issued
    bool ok = true;
    for (int base = 0; base < count && ok; base += 16) {
      // block ids of items base .. base + 15, two per item (lane 2 q + h: item q, half h)
      int my_blk = -1;
      {
        ItemWalk w2 = it;
        for (int q = 0; q < (lane >> 1); ++q) w2.next(a);
        if (base + (lane >> 1) < count) {
          const int tb = w2.j * kITok + (lane & 1) * kIBlk;
          if (tb < row_tokens(a, w2.r, false)) {
            const int v = __ldg(a.block_table + (size_t)(w2.r / a.Sq) * a.max_blocks + tb / kIBlk);
            my_blk = (v >= 0 && v < a.num_blocks) ? v : -2;
          }
        }
      }
      const int nq = min(16, count - base);
      for (int q = 0; q < nq && ok; ++q, it.next(a)) {
        const int blk0 = __shfl_sync(0xffffffffu, my_blk, 2 * q), blk1 = __shfl_sync(0xffffffffu, my_blk, 2 * q + 1);
        const int i = base + q;
        if (it.r != cur_row) {   // the row's query, head scales and weights into the next slot
          cur_row = it.r;
          ++rs;
          const uint32_t slot = rs & 1;
          if (lane == 0) ok = mbar_wait<false>(smem_u32(&ctl.q_empty[slot]), ((rs >> 1) & 1) ^ 1, abort, timeout_ns);
          ok = __shfl_sync(0xffffffffu, ok, 0);
          if (!ok) break;
          for (int h = lane; h < kDsaHeads; h += 32)
            ctl.wq[slot][h] = __ldg(a.w + (size_t)cur_row * kDsaHeads + h) *
                              __ldg(a.q_scale + (size_t)cur_row * kDsaHeads + h);
          __syncwarp();
          if (lane == 0) {
            mbar_arrive_expect_tx(smem_u32(&ctl.q_full[slot]), kIQ);   // releases the warp's stores above
            tma_load_2d(sQ + slot * kIQ, &tm_q, smem_u32(&ctl.q_full[slot]), 0, cur_row * kDsaHeads);
          }
        }
        if (lane == 0) {
          if (blk0 == -2 || blk1 == -2) set_status(a.status, MLA_ERR_BAD_BLOCK_ID);
          const uint32_t st = i % kIStages;
          ok = mbar_wait<false>(smem_u32(&ctl.empty[st]), ((i / kIStages) & 1) ^ 1, abort, timeout_ns);
          if (ok) {
            const uint32_t bar = smem_u32(&ctl.full[st]);
            constexpr uint32_t kBlkBytes = kIBlk * kDsaDim + kIBlk * 4;   // codes + scales of one block
            ctl.valid[st] = (blk0 >= 0 ? 1u : 0u) | (blk1 >= 0 ? 2u : 0u);   // released by the arrive below
            mbar_arrive_expect_tx(bar, (blk0 >= 0 ? kBlkBytes : 0u) + (blk1 >= 0 ? kBlkBytes : 0u));
            if (blk0 >= 0) {
              tma_load_3d(sK + st * kIKTile, &tm_k, bar, 0, 0, blk0);
              tma_load_2d(sS + st * kIScales, &tm_s, bar, 0, blk0);
            }
            if (blk1 >= 0) {
              tma_load_3d(sK + st * kIKTile + kIBlk * kDsaDim, &tm_k, bar, 0, 0, blk1);
              tma_load_2d(sS + st * kIScales + kIBlk * 4, &tm_s, bar, 0, blk1);
            }
            ++issued;
          }
        }
        ok = __shfl_sync(0xffffffffu, ok, 0);
      }
    }
    if (lane == 0) {
      // every load issued lands before the CTA may exit
      int dummy = 0;
      for (int i = max(0, issued - kIStages); i < issued; ++i)
        mbar_wait<false>(smem_u32(&ctl.full[i % kIStages]), (i / kIStages) & 1, &dummy, drain_ns);
      if (!ok) {
        set_status(a.status, MLA_ERR_TIMEOUT);
        *abort = 1;
      }
    }
  } else if (warp == kIMma) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3_f32(kITok, kDsaHeads);
      ItemWalk it;
      it.start(a, ctl.r0, ctl.j0);
      int cur_row = -1, rs = -1;
      bool ok = true;
      for (int i = 0; i < count && ok; ++i) {
        if (it.r != cur_row) {
          cur_row = it.r;
          ++rs;
          ok = mbar_wait<false>(smem_u32(&ctl.q_full[rs & 1]), (rs >> 1) & 1, abort, timeout_ns);
          if (!ok) break;
        }
        const uint32_t st = i % kIStages, ac = i % kIAcc;
        ok = mbar_wait<false>(smem_u32(&ctl.full[st]), (i / kIStages) & 1, abort, timeout_ns) &&
             mbar_wait<false>(smem_u32(&ctl.acc_empty[ac]), ((i / kIAcc) & 1) ^ 1, abort, timeout_ns);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < kDsaDim / 32; ++kk) {
          // 32 codes = 32 bytes of every 128-byte row per step (K-major, 128-byte swizzle)
          const uint64_t ad = smem_desc(sK + st * kIKTile + kk * 32, 16, 1024, kSwizzle128B);
          const uint64_t bd = smem_desc(sQ + (rs & 1) * kIQ + kk * 32, 16, 1024, kSwizzle128B);
          mma_f8_ss(tmem + kDsaHeads * ac, ad, bd, idesc, kk ? 1u : 0u);
        }
        mma_commit(smem_u32(&ctl.empty[st]));
        mma_commit(smem_u32(&ctl.acc_full[ac]));
        ItemWalk nx = it;
        nx.next(a);
        if (i + 1 == count || nx.r != cur_row) mma_commit(smem_u32(&ctl.q_empty[rs & 1]));   // query slot free
        it = nx;
      }
      if (!ok) {
        set_status(a.status, MLA_ERR_TIMEOUT);
        *abort = 1;
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (thread = token row)
    // TMEM lane quarter = warp % 4 in both groups; group g takes the items of parity g
    const int grp = warp < 4 ? 0 : 1;
    const int quarter = warp & 3;
    ItemWalk it;
    it.start(a, ctl.r0, ctl.j0);
    int cur_row = -1, rs = -1, n = 0;
    const int tr = quarter * 32 + lane;
    const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
    bool ok = true;
    for (int i = 0; i < count && ok; ++i, it.next(a)) {
      if (it.r != cur_row) {   // done with the previous row's slot; the new row's scales and weights
        if (rs >= 0 && lane == 0) mbar_arrive(smem_u32(&ctl.q_empty[rs & 1]));
        cur_row = it.r;
        ++rs;
        n = row_tokens(a, cur_row, false);
        int dummy = 0;
        ok = __all_sync(0xffffffffu, mbar_wait<false>(smem_u32(&ctl.q_full[rs & 1]), (rs >> 1) & 1, &dummy,
                                                      timeout_ns) && !*abort);
        if (!ok) break;
      }
      if (kIGroups == 2 && (i & 1) != grp) continue;   // the other group's item
      const float* wq = ctl.wq[rs & 1];
      const int t = it.j * kITok + tr;
      const uint32_t st = i % kIStages, ac = i % kIAcc;
      int dummy = 0;
      // the stage's key scales and validity (TMA), then the accumulator; warp-uniform waits:
      // the TMEM loads below are warp-collective
      ok = __all_sync(0xffffffffu, mbar_wait<false>(smem_u32(&ctl.full[st]), (i / kIStages) & 1, &dummy,
                                                    timeout_ns) && !*abort);
      if (!ok) break;
      const bool valid = (ctl.valid[st] >> (tr / kIBlk)) & 1u;
      const float ks = scale_ring[st * kITok + tr];
      ok = __all_sync(0xffffffffu, mbar_wait<false>(smem_u32(&ctl.acc_full[ac]), (i / kIAcc) & 1, &dummy,
                                                    timeout_ns) && !*abort);
      if (!ok) break;
      tc_fence_after();
      uint32_t v[kDsaHeads];
#pragma unroll
      for (int c = 0; c < kDsaHeads / 16; ++c) tmem_ld16(tmem + lane_off + kDsaHeads * ac + 16 * c, v + 16 * c);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(smem_u32(&ctl.acc_empty[ac]));
        mbar_arrive(smem_u32(&ctl.empty[st]));   // this warp is done with the stage's scales
      }
      if (t < n) {
        // scales are >= 0, so ReLU(w q_s k_s dot) = k_s * w q_s * ReLU(dot); four partial sums
        float p[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int j = 0; j < kDsaHeads; ++j) p[j & 3] = fmaf(wq[j], fmaxf(__uint_as_float(v[j]), 0.f), p[j & 3]);
        const float I = valid ? ks * ((p[0] + p[1]) + (p[2] + p[3])) : __int_as_float(0x7fc00000);   // NaN: bad block
        a.scores[(size_t)cur_row * a.max_seq_len + t] = I;
      }
    }
    if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
    if (ok && rs >= 0 && lane == 0) mbar_arrive(smem_u32(&ctl.q_empty[rs & 1]));
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kIMma) {
    tc_fence_after();
    tmem_dealloc(tmem, kITmemCols);
  }
}

// -------------------------------------------------------------------------------- top-k
constexpr int kTkThreads = 1024;
constexpr int kTkCluster = 8;                  // CTAs per query row
constexpr int kTkPer = 8;                      // consecutive positions per thread, ordered pass
constexpr int kTkReg = 16;                     // keys per thread kept in registers (slices up to 16384)

// order-preserving unsigned key of an fp32 score; -0 and +0 share one key
__device__ __forceinline__ uint32_t score_key(float x) {
  uint32_t u = __float_as_uint(x);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// exclusive block-wide prefix sum of a 64-bit value (1024 threads); *total = the sum
__device__ __forceinline__ uint64_t block_scan_excl(uint64_t v, uint64_t* wsum, uint64_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wsum[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint64_t t = wsum[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint64_t y = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += y;
    }
    wsum[lane] = t;
  }
  __syncthreads();
  const uint64_t ex = x - v + (warp ? wsum[warp - 1] : 0ull);
  *total = wsum[31];
  __syncthreads();
  return ex;
}

// distributed shared memory: a 32-bit word of a cluster peer's shared memory
__device__ __forceinline__ uint32_t ld_dsmem_u32(uint32_t cluster_addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(cluster_addr) : "memory");
  return v;
}
__device__ __forceinline__ void st_dsmem_u32(uint32_t cluster_addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(cluster_addr), "r"(v) : "memory");
}

// One cluster of kTkCluster CTAs per query row; CTA `rank` owns the slice
// [n rank / C, n (rank + 1) / C) of the row's scores. Histograms are summed by rank 0 through
// distributed shared memory, which broadcasts each pass's digit; the ordered pass writes
// each slice at offsets given by the counts of the lower ranks.
__global__ void __cluster_dims__(kTkCluster, 1, 1) __launch_bounds__(kTkThreads, 1) dsa_topk_kernel(const DsaArgs a) {
  __shared__ uint32_t hist[2048];
  __shared__ uint64_t wsum[32];
  __shared__ uint32_t pick[2];     // written by rank 0 into every CTA of the cluster
  __shared__ uint32_t slice[2];    // this slice's counts above and equal to the threshold key
  const int tid = threadIdx.x;
  const uint32_t rank = cluster_ctarank();
  const int row = blockIdx.x / kTkCluster, b = row / a.Sq, s = row % a.Sq;
  const int k = a.top_k;
  int L = __ldg(a.seq_lens + b);
  if (L < 0 || L > a.max_blocks * a.bs || L > a.max_seq_len) {
    if (tid == 0 && rank == 0) set_status(a.status, MLA_ERR_BAD_SEQ_LEN);
    L = 0;
  }
  const int n = max(a.causal ? L - a.Sq + 1 + s : L, 0);
  int32_t* out = a.indices + (size_t)row * k;
  if (n <= k) {   // every candidate is kept (the same branch in every CTA of the cluster)
    for (int j = (int)rank * kTkThreads + tid; j < k; j += kTkThreads * kTkCluster) out[j] = j < n ? j : -1;
    if (tid == 0 && rank == 0) a.counts[row] = n;
    return;
  }
  const float* sc = a.scores + (size_t)row * a.max_seq_len;
  const int lo = (int)((long long)n * rank / kTkCluster), hi = (int)((long long)n * (rank + 1) / kTkCluster);
  // the slice's keys stay in registers when they fit (element j of a thread: lo + j 1024 + tid)
  const bool in_regs = hi - lo <= kTkThreads * kTkReg;
  uint32_t kr[kTkReg];
#pragma unroll
  for (int j = 0; j < kTkReg; ++j) {
    const int i = lo + j * kTkThreads + tid;
    kr[j] = (in_regs && i < hi) ? score_key(__ldg(sc + i)) : 0u;
  }
  auto for_each_key = [&](auto&& f) {
    if (in_regs) {
#pragma unroll
      for (int j = 0; j < kTkReg; ++j)
        if (lo + j * kTkThreads + tid < hi) f(kr[j]);
    } else {
      for (int i = lo + tid; i < hi; i += kTkThreads) f(score_key(__ldg(sc + i)));
    }
  };

  // radix select of the k-th largest key: after the passes, T = prefix and `rem` entries
  // equal to T are kept (the rest of the k are above T)
  uint32_t prefix = 0, pmask = 0, rem = (uint32_t)k;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    // key bits [21, 32), [10, 21), [0, 10)
    const int shift = pass == 0 ? 21 : pass == 1 ? 10 : 0, nb = pass == 2 ? 1024 : 2048;
    const uint32_t dmask = (uint32_t)nb - 1u;
    for (int i = tid; i < 2048; i += kTkThreads) hist[i] = 0u;
    __syncthreads();
    for_each_key([&](uint32_t key) {
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
    });
    cluster_sync();   // every slice's histogram is complete
    if (rank == 0) {
      // digits in descending order, two per thread: where does the running count reach rem?
      const int d_hi = nb - 1 - 2 * tid, d_lo = nb - 2 - 2 * tid;
      // all remote loads first, then the sums (the loads overlap)
      uint32_t h_hi[kTkCluster], h_lo[kTkCluster];
#pragma unroll
      for (uint32_t r = 0; r < kTkCluster; ++r) {
        h_hi[r] = d_hi >= 0 ? ld_dsmem_u32(mapa(smem_u32(&hist[d_hi]), r)) : 0u;
        h_lo[r] = d_lo >= 0 ? ld_dsmem_u32(mapa(smem_u32(&hist[d_lo]), r)) : 0u;
      }
      uint32_t c_hi = 0, c_lo = 0;
#pragma unroll
      for (uint32_t r = 0; r < kTkCluster; ++r) {
        c_hi += h_hi[r];
        c_lo += h_lo[r];
      }
      uint64_t tot;
      const uint32_t above = (uint32_t)block_scan_excl((uint64_t)(c_hi + c_lo), wsum, &tot);
      uint32_t d = 0xffffffffu, ab = 0;
      if (above < rem && rem <= above + c_hi) {
        d = (uint32_t)d_hi;
        ab = above;
      } else if (above + c_hi < rem && rem <= above + c_hi + c_lo) {
        d = (uint32_t)d_lo;
        ab = above + c_hi;
      }
      if (d != 0xffffffffu)
        for (uint32_t r = 0; r < kTkCluster; ++r) {
          st_dsmem_u32(mapa(smem_u32(&pick[0]), r), d);
          st_dsmem_u32(mapa(smem_u32(&pick[1]), r), ab);
        }
    }
    cluster_sync();   // the pick is everywhere; rank 0 is done reading the histograms
    rem -= pick[1];
    prefix |= pick[0] << shift;
    pmask |= dmask << shift;
  }
  const uint32_t T = prefix;

  // this slice's counts, then its offsets: the counts of the lower ranks
  {
    uint32_t gt = 0, tie = 0;
    for_each_key([&](uint32_t key) {
      gt += key > T ? 1u : 0u;
      tie += key == T ? 1u : 0u;
    });
    uint64_t tot;
    block_scan_excl(((uint64_t)gt << 32) | tie, wsum, &tot);
    if (tid == 0) {
      slice[0] = (uint32_t)(tot >> 32);
      slice[1] = (uint32_t)(tot & 0xffffffffu);
    }
  }
  cluster_sync();
  uint32_t run_gt = 0, run_tie = 0;
  {
    uint32_t g8[kTkCluster], t8[kTkCluster];
#pragma unroll
    for (uint32_t r = 0; r < kTkCluster; ++r) {
      g8[r] = r < rank ? ld_dsmem_u32(mapa(smem_u32(&slice[0]), r)) : 0u;
      t8[r] = r < rank ? ld_dsmem_u32(mapa(smem_u32(&slice[1]), r)) : 0u;
    }
#pragma unroll
    for (uint32_t r = 0; r < kTkCluster; ++r) {
      run_gt += g8[r];
      run_tie += t8[r];
    }
  }

  // ordered pass: positions above T, and the first `rem` positions equal to T
#pragma unroll 1
  for (int base = lo; base < hi; base += kTkThreads * kTkPer) {
    const int p0 = base + tid * kTkPer;
    uint32_t keys[kTkPer];
    uint32_t gt = 0, tie = 0;
#pragma unroll
    for (int m = 0; m < kTkPer; ++m) {
      const bool valid = p0 + m < hi;
      keys[m] = valid ? score_key(__ldg(sc + p0 + m)) : 0u;
      gt += (valid && keys[m] > T) ? 1u : 0u;
      tie += (valid && keys[m] == T) ? 1u : 0u;
    }
    uint64_t tot;
    const uint64_t ex = block_scan_excl(((uint64_t)gt << 32) | tie, wsum, &tot);
    uint32_t g_before = run_gt + (uint32_t)(ex >> 32), t_before = run_tie + (uint32_t)(ex & 0xffffffffu);
#pragma unroll
    for (int m = 0; m < kTkPer; ++m) {
      if (p0 + m >= hi) break;
      if (keys[m] > T) {
        out[g_before + min(t_before, rem)] = p0 + m;
        ++g_before;
      } else if (keys[m] == T) {
        if (t_before < rem) out[g_before + t_before] = p0 + m;
        ++t_before;
      }
    }
    run_gt += (uint32_t)(tot >> 32);
    run_tie += (uint32_t)(tot & 0xffffffffu);
  }
  if (tid == 0 && rank == 0) a.counts[row] = k;
  cluster_sync();   // no CTA leaves while a peer may still read its shared memory
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

// byte-element tensor map, 128-byte swizzle: rank 2 or 3, dims inner -> outer
bool map_u8(CUtensorMap* m, const void* base, int rank, const cuuint64_t* dims, const cuuint64_t* strides,
            const cuuint32_t* box) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, rank, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

cudaError_t launch_dsa_index(const DsaArgs& a, cudaStream_t s) {
  const int R = a.B * a.Sq;
  if (R == 0 || a.max_seq_len == 0) return cudaSuccess;
  CUtensorMap tq, tk, ts;
  // query codes [R * 64 rows][128 B], box 64 rows; key codes [num_blocks][64][128 B], box one block
  const cuuint64_t qd[2] = {(cuuint64_t)kDsaDim, (cuuint64_t)R * kDsaHeads};
  const cuuint64_t qs[1] = {(cuuint64_t)kDsaDim};
  const cuuint32_t qb[2] = {(cuuint32_t)kDsaDim, (cuuint32_t)kDsaHeads};
  const cuuint64_t kd[3] = {(cuuint64_t)kDsaDim, (cuuint64_t)kIBlk, (cuuint64_t)a.num_blocks};
  const cuuint64_t ks[2] = {(cuuint64_t)kDsaDim, (cuuint64_t)kIBlk * kDsaDim};
  const cuuint32_t kb[3] = {(cuuint32_t)kDsaDim, (cuuint32_t)kIBlk, 1};
  if (!map_u8(&tq, a.q, 2, qd, qs, qb) || !map_u8(&tk, a.k, 3, kd, ks, kb)) return cudaErrorInvalidValue;
  {
    // key scales [num_blocks][64] f32, box one block
    EncodeTiledFn fn = encode_fn();
    const cuuint64_t sd[2] = {(cuuint64_t)kIBlk, (cuuint64_t)a.num_blocks};
    const cuuint64_t ss[1] = {(cuuint64_t)kIBlk * 4};
    const cuuint32_t sb[2] = {(cuuint32_t)kIBlk, 1};
    const cuuint32_t estr[2] = {1, 1};
    if (!fn || fn(&ts, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(a.k_scale), sd, ss, sb, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return cudaErrorInvalidValue;
  }
  static std::once_flag attr_once[64];
  static int sms[64];
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t err = cudaSuccess;
  std::call_once(attr_once[dev & 63], [&] {
    err = cudaFuncSetAttribute(dsa_index_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kISmem);
    if (err == cudaSuccess) err = cudaDeviceGetAttribute(&sms[dev & 63], cudaDevAttrMultiProcessorCount, dev);
  });
  if (err != cudaSuccess) return err;
  // kICtasPerSm CTAs per SM, fewer when there are fewer tiles
  const long long tiles_max = (long long)R * ((a.max_seq_len + kITok - 1) / kITok);
  const int grid = (int)std::min<long long>((long long)kICtasPerSm * std::max(sms[dev & 63], 1), std::max(tiles_max, 1ll));
  dsa_index_kernel<<<grid, kIThreads, kISmem, s>>>(tq, tk, ts, a, wait_timeout_ns(), drain_timeout_ns());
  return cudaGetLastError();
}

cudaError_t launch_dsa_topk(const DsaArgs& a, cudaStream_t s) {
  const int R = a.B * a.Sq;
  if (R == 0) return cudaSuccess;
  dsa_topk_kernel<<<R * kTkCluster, kTkThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace mla
