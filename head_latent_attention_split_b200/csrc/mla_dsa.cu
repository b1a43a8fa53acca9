// DeepSeek Sparse Attention side kernels ("TransMLA & Sparse Latent Attention" lesson,
// Chapter 6 "The lightning indexer" and "Fine-grained token selection"; Chapter 7 "Why
// FP8 specifically" and "The indexer keeps its own small cache").
//
// Indexer: I_t = sum_j w_j * ReLU(q_j . k_t) for every token t a query row may see, with
// H^I = 64 heads of width d^I = 128 stored as e4m3 codes with one fp32 scale per vector
// (q per head, k per cached token). One CTA = one query row and up to four 128-token
// tiles. TMA brings the row's 64 x 128 query codes and each tile's key codes (two cache
// blocks, 128-byte swizzled); one thread issues tcgen05 MMAs of kind::f8f6f4 with the
// tokens as M = 128 and the heads as N = 64 (K = 4 x 32 codes), so every TMEM lane holds
// one token's 64 head dots and the thread reading it finishes that token alone: scale,
// ReLU, weighted sum, one coalesced fp32 store. The e4m3 products are exact and summed in
// fp32 by the tensor core.
//
// Top-k: one 1024-thread CTA per query row. A three-pass radix select (11, 11, 10 bits of
// an order-preserving key of the fp32 score) finds the k-th largest key T and how many
// entries equal to T are kept; one ordered pass then writes the positions of every score
// above T and of the first such ties, in ascending position order (a block-wide scan of
// packed counts). Ties at T go to the lower positions, so the result is unique.
#include <cuda.h>

#include <mutex>

#include "mla_device.cuh"
#include "ptx_sm100.cuh"

namespace mla {
namespace {

using namespace ptx;

// ------------------------------------------------------------------------------ indexer
constexpr int kITok = 128;                        // tokens per tile = MMA M
constexpr int kITiles = 4;                        // tiles per CTA
constexpr int kIBlk = 64;                         // tokens per cache block
constexpr uint32_t kIKTile = kITok * kDsaDim;     // 16 KB of key codes
constexpr uint32_t kIQ = kDsaHeads * kDsaDim;     // 8 KB of query codes
constexpr uint32_t kITmemCols = kITiles * kDsaHeads;   // one 64-column accumulator per tile

struct IdxCtl {
  uint64_t full[kITiles];
  uint64_t done[kITiles];
  uint64_t q_full;
  uint32_t tmem_base;
  int abort;
  uint32_t blocks[kITiles][2];   // cache block of each 64-token half, or ~0u if not loaded
  float qs[kDsaHeads];
  float w[kDsaHeads];
};
// Two CTAs per SM: their accumulators (2 x 256 TMEM columns) fill the SM's 512, so the
// request is sized to keep a third from being placed (it would wait in the allocator).
constexpr uint32_t kISmem = 104 * 1024;
static_assert(kITiles * kIKTile + kIQ + 1024 + 1024 <= kISmem && 3 * kISmem > 232448, "indexer shared memory");
static_assert(sizeof(IdxCtl) <= 1024, "indexer control block");

__global__ void __launch_bounds__(128, 1)
    dsa_index_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const DsaArgs a, const uint64_t timeout_ns) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  IdxCtl& ctl = *reinterpret_cast<IdxCtl*>(smem + kITiles * kIKTile + kIQ);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int row = blockIdx.y;                       // query row (b, s)
  const int b = row / a.Sq, s = row % a.Sq;
  const int cap = a.max_blocks * a.bs;
  int L = __ldg(a.seq_lens + b);
  if (L < 0 || L > cap || L > a.max_seq_len) {
    if (threadIdx.x == 0 && blockIdx.x == 0) set_status(a.status, MLA_ERR_BAD_SEQ_LEN);
    return;
  }
  const int n = max(a.causal ? L - a.Sq + 1 + s : L, 0);   // tokens this row sees
  const int t0 = blockIdx.x * kITiles * kITok;
  if (t0 >= n) return;                                     // the whole CTA
  const int ntile = min(kITiles, (n - t0 + kITok - 1) / kITok);
  const uint32_t sK = smem_u32(smem), sQ = smem_u32(smem + kITiles * kIKTile);
  volatile int* abort = &ctl.abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kITiles; ++i) {
      mbar_init(smem_u32(&ctl.full[i]), 1);
      mbar_init(smem_u32(&ctl.done[i]), 1);
    }
    mbar_init(smem_u32(&ctl.q_full), 1);
    ctl.abort = 0;
    fence_mbarrier_init_cluster();
  }
  if (threadIdx.x < kDsaHeads) {
    ctl.qs[threadIdx.x] = __ldg(a.q_scale + (size_t)row * kDsaHeads + threadIdx.x);
    ctl.w[threadIdx.x] = __ldg(a.w + (size_t)row * kDsaHeads + threadIdx.x);
  } else if (threadIdx.x < kDsaHeads + 2 * kITiles) {
    // the cache block of each 64-token half of each tile (~0u: past the row or invalid)
    const int i = (threadIdx.x - kDsaHeads) >> 1, h = (threadIdx.x - kDsaHeads) & 1;
    const int tb = t0 + i * kITok + h * kIBlk;
    uint32_t blk = ~0u;
    if (i < ntile && tb < n) {
      const int v = __ldg(a.block_table + (size_t)b * a.max_blocks + tb / kIBlk);
      if (v >= 0 && v < a.num_blocks)
        blk = (uint32_t)v;
      else
        set_status(a.status, MLA_ERR_BAD_BLOCK_ID);
    }
    ctl.blocks[i][h] = blk;
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&ctl.tmem_base), kITmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;

  if (threadIdx.x == 0) {
    // loads: the query, then each tile's (up to) two cache blocks
    mbar_arrive_expect_tx(smem_u32(&ctl.q_full), kIQ);
    tma_load_2d(sQ, &tm_q, smem_u32(&ctl.q_full), 0, row * kDsaHeads);
    for (int i = 0; i < ntile; ++i) {
      const uint32_t bytes = (ctl.blocks[i][0] != ~0u ? kIBlk * kDsaDim : 0u) + (ctl.blocks[i][1] != ~0u ? kIBlk * kDsaDim : 0u);
      const uint32_t bar = smem_u32(&ctl.full[i]);
      mbar_arrive_expect_tx(bar, bytes);
      for (int h = 0; h < 2; ++h)
        if (ctl.blocks[i][h] != ~0u)
          tma_load_3d(sK + i * kIKTile + h * (kIBlk * kDsaDim), &tm_k, bar, 0, 0, (int)ctl.blocks[i][h]);
    }
    // MMAs: tile i -> accumulator columns [64 i, 64 i + 64)
    constexpr uint32_t idesc = idesc_e4m3_f32(kITok, kDsaHeads);
    bool ok = mbar_wait<false>(smem_u32(&ctl.q_full), 0, abort, timeout_ns);
    for (int i = 0; i < ntile && ok; ++i) {
      ok = mbar_wait<false>(smem_u32(&ctl.full[i]), 0, abort, timeout_ns);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < kDsaDim / 32; ++kk) {
        // 32 codes = 32 bytes of every 128-byte row per step (K-major, 128-byte swizzle)
        const uint64_t ad = smem_desc(sK + i * kIKTile + kk * 32, 16, 1024, kSwizzle128B);
        const uint64_t bd = smem_desc(sQ + kk * 32, 16, 1024, kSwizzle128B);
        mma_f8_ss(tmem + kDsaHeads * i, ad, bd, idesc, kk ? 1u : 0u);
      }
      mma_commit(smem_u32(&ctl.done[i]));
    }
    if (!ok) {
      set_status(a.status, MLA_ERR_TIMEOUT);
      ctl.abort = 1;
    }
  }

  // epilogue: thread = token row of the tile (TMEM lane 32 warp + lane)
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  bool ok = true;
  for (int i = 0; i < ntile && ok; ++i) {
    int dummy = 0;
    // warp-uniform: the TMEM loads below are warp-collective
    ok = __all_sync(0xffffffffu, mbar_wait<false>(smem_u32(&ctl.done[i]), 0, &dummy, timeout_ns) && !*abort);
    if (!ok) break;
    tc_fence_after();
    uint32_t v[kDsaHeads];
#pragma unroll
    for (int c = 0; c < kDsaHeads / 16; ++c) tmem_ld16(tmem + lane_off + kDsaHeads * i + 16 * c, v + 16 * c);
    tmem_wait_ld();
    const int tr = warp * 32 + lane;                 // row of the tile
    const int t = t0 + i * kITok + tr;
    if (t < n) {
      const uint32_t blk = ctl.blocks[i][tr / kIBlk];
      float I = __int_as_float(0x7fc00000);          // NaN where the block id was invalid
      if (blk != ~0u) {
        const float ks = __ldg(a.k_scale + (size_t)blk * kIBlk + (tr % kIBlk));
        I = 0.f;
#pragma unroll
        for (int j = 0; j < kDsaHeads; ++j) I = fmaf(ctl.w[j], fmaxf(__uint_as_float(v[j]) * (ctl.qs[j] * ks), 0.f), I);
      }
      a.scores[(size_t)row * a.max_seq_len + t] = I;
    }
  }
  if (!ok) set_status(a.status, MLA_ERR_TIMEOUT);
  // every load issued has landed before the CTA may exit
  if (threadIdx.x == 0) {
    int dummy = 0;
    mbar_wait<false>(smem_u32(&ctl.q_full), 0, &dummy, timeout_ns);
    for (int i = 0; i < ntile; ++i) mbar_wait<false>(smem_u32(&ctl.full[i]), 0, &dummy, timeout_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kITmemCols);
  }
}

// -------------------------------------------------------------------------------- top-k
constexpr int kTkThreads = 1024;
constexpr int kTkPer = 8;                      // consecutive positions per thread, ordered pass

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

__global__ void __launch_bounds__(kTkThreads, 1) dsa_topk_kernel(const DsaArgs a) {
  __shared__ uint32_t hist[2048];
  __shared__ uint64_t wsum[32];
  __shared__ uint32_t pick[2];
  const int tid = threadIdx.x;
  const int row = blockIdx.x, b = row / a.Sq, s = row % a.Sq;
  const int k = a.top_k;
  int L = __ldg(a.seq_lens + b);
  if (L < 0 || L > a.max_blocks * a.bs || L > a.max_seq_len) {
    if (tid == 0) set_status(a.status, MLA_ERR_BAD_SEQ_LEN);
    L = 0;
  }
  const int n = max(a.causal ? L - a.Sq + 1 + s : L, 0);
  int32_t* out = a.indices + (size_t)row * k;
  if (n <= k) {   // every candidate is kept
    for (int j = tid; j < k; j += kTkThreads) out[j] = j < n ? j : -1;
    if (tid == 0) a.counts[row] = n;
    return;
  }
  const float* sc = a.scores + (size_t)row * a.max_seq_len;

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
    for (int i = tid; i < n; i += kTkThreads) {
      const uint32_t key = score_key(__ldg(sc + i));
      if ((key & pmask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
    }
    __syncthreads();
    // digits in descending order, two per thread: where does the running count reach rem?
    const int d_hi = nb - 1 - 2 * tid, d_lo = nb - 2 - 2 * tid;
    const uint32_t c_hi = d_hi >= 0 ? hist[d_hi] : 0u, c_lo = d_lo >= 0 ? hist[d_lo] : 0u;
    uint64_t tot;
    const uint32_t above = (uint32_t)block_scan_excl((uint64_t)(c_hi + c_lo), wsum, &tot);
    if (above < rem && rem <= above + c_hi) {
      pick[0] = (uint32_t)d_hi;
      pick[1] = above;
    } else if (above + c_hi < rem && rem <= above + c_hi + c_lo) {
      pick[0] = (uint32_t)d_lo;
      pick[1] = above + c_hi;
    }
    __syncthreads();
    rem -= pick[1];
    prefix |= pick[0] << shift;
    pmask |= dmask << shift;
    __syncthreads();
  }
  const uint32_t T = prefix;

  // ordered pass: positions above T, and the first `rem` positions equal to T
  uint32_t run_gt = 0, run_tie = 0;
#pragma unroll 1
  for (int base = 0; base < n; base += kTkThreads * kTkPer) {
    const int p0 = base + tid * kTkPer;
    uint32_t keys[kTkPer];
    uint32_t gt = 0, tie = 0;
#pragma unroll
    for (int m = 0; m < kTkPer; ++m) {
      keys[m] = p0 + m < n ? score_key(__ldg(sc + p0 + m)) : 0u;
      const bool valid = p0 + m < n;
      gt += (valid && keys[m] > T) ? 1u : 0u;
      tie += (valid && keys[m] == T) ? 1u : 0u;
    }
    uint64_t tot;
    const uint64_t ex = block_scan_excl(((uint64_t)gt << 32) | tie, wsum, &tot);
    uint32_t g_before = run_gt + (uint32_t)(ex >> 32), t_before = run_tie + (uint32_t)(ex & 0xffffffffu);
#pragma unroll
    for (int m = 0; m < kTkPer; ++m) {
      if (p0 + m >= n) break;
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
  if (tid == 0) a.counts[row] = k;
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
  CUtensorMap tq, tk;
  // query codes [R * 64 rows][128 B], box 64 rows; key codes [num_blocks][64][128 B], box one block
  const cuuint64_t qd[2] = {(cuuint64_t)kDsaDim, (cuuint64_t)R * kDsaHeads};
  const cuuint64_t qs[1] = {(cuuint64_t)kDsaDim};
  const cuuint32_t qb[2] = {(cuuint32_t)kDsaDim, (cuuint32_t)kDsaHeads};
  const cuuint64_t kd[3] = {(cuuint64_t)kDsaDim, (cuuint64_t)kIBlk, (cuuint64_t)a.num_blocks};
  const cuuint64_t ks[2] = {(cuuint64_t)kDsaDim, (cuuint64_t)kIBlk * kDsaDim};
  const cuuint32_t kb[3] = {(cuuint32_t)kDsaDim, (cuuint32_t)kIBlk, 1};
  if (!map_u8(&tq, a.q, 2, qd, qs, qb) || !map_u8(&tk, a.k, 3, kd, ks, kb)) return cudaErrorInvalidValue;
  static std::once_flag attr_once[64];
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t err = cudaSuccess;
  std::call_once(attr_once[dev & 63], [&] {
    err = cudaFuncSetAttribute(dsa_index_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kISmem);
  });
  if (err != cudaSuccess) return err;
  const dim3 grid((a.max_seq_len + kITiles * kITok - 1) / (kITiles * kITok), R);
  dsa_index_kernel<<<grid, 128, kISmem, s>>>(tq, tk, a, 2000000000ull);
  return cudaGetLastError();
}

cudaError_t launch_dsa_topk(const DsaArgs& a, cudaStream_t s) {
  const int R = a.B * a.Sq;
  if (R == 0) return cudaSuccess;
  dsa_topk_kernel<<<R, kTkThreads, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace mla
