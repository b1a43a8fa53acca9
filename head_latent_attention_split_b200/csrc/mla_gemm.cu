// Per-head GEMM around the decode: y[m, h, :] = x[m, h, :] . w[h] for every head h, bf16
// operands, fp32 accumulation in TMEM, bf16 result. With w = W^UK (d_h x r) it is the
// query absorption, with w = W^UV^T (r x d_v) the output up-projection ("TransMLA:
// Multi-Head Latent Attention Is All You Need", sec. 3.4.5: W^UK is absorbed into the
// query and W^UV into the output side). See mla_head_gemm in include/mla_decode.h.
//
// One CTA per (N tile of up to 256 columns, head, 128 rows): TMA loads 64-wide K chunks of
// x (rows of head h, K-major, 128-byte swizzle) and w[h] (N-major, 64-column chunks) into a
// two-stage ring; one thread issues tcgen05 MMAs (M = 128, K = 16) into a TMEM accumulator;
// four warps read it back (one row per thread), round to bf16 and store the valid rows.
#include <cuda.h>

#include <mutex>

#include "mla_device.cuh"
#include "ptx_sm100.cuh"

namespace mla {
namespace {

using namespace ptx;

constexpr int kGM = 128;                 // rows per CTA = MMA M
constexpr int kGK = 64;                  // K per chunk: one 128-byte swizzled row of bf16
constexpr uint32_t kAChunk = kGM * 128;  // [128 rows][64 k] bf16
constexpr uint32_t kBChunk = kGK * 128;  // [64 k][64 n] bf16, one of ntile / 64 per stage

// two fp32 -> bf16x2 (lo in the low half), round to nearest even
__device__ __forceinline__ uint32_t pack2_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

struct GemmCtl {
  uint64_t full[2], empty[2], done;
  uint32_t tmem_base;
  int abort;
};

template <int kNT>
__global__ void __launch_bounds__(128, 1)
    head_gemm_kernel(const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_w,
                     const GemmArgs a, const uint64_t timeout_ns, const uint64_t drain_ns) {
  constexpr uint32_t kStage = kAChunk + (kNT / 64) * kBChunk;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = (uint8_t*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  GemmCtl& ctl = *reinterpret_cast<GemmCtl*>(smem + 2 * kStage);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * kNT, h = blockIdx.y, m0 = blockIdx.z * kGM;
  const int nk = a.k / kGK;
  volatile int* abort = &ctl.abort;
  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(smem_u32(&ctl.full[i]), 1);
      mbar_init(smem_u32(&ctl.empty[i]), 1);
    }
    mbar_init(smem_u32(&ctl.done), 1);
    ctl.abort = 0;
    fence_mbarrier_init_cluster();
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(&ctl.tmem_base), kNT < 32 ? 32 : kNT);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = ctl.tmem_base;
  bool ok = true;
  if (threadIdx.x == 0) {
    auto load = [&](int kc) {
      const uint32_t st = kc & 1;
      const uint32_t base = smem_u32(smem + st * kStage);
      const uint32_t bar = smem_u32(&ctl.full[st]);
      mbar_arrive_expect_tx(bar, kStage);
      tma_load_3d(base, &tm_x, bar, kc * kGK, h, m0);
#pragma unroll
      for (int j = 0; j < kNT / 64; ++j) tma_load_3d(base + kAChunk + j * kBChunk, &tm_w, bar, n0 + 64 * j, kc * kGK, h);
    };
    constexpr uint32_t idesc = idesc_bf16_f32(kGM, kNT, true);
    load(0);
    if (nk > 1) load(1);
    for (int kc = 0; kc < nk && ok; ++kc) {
      const uint32_t st = kc & 1;
      ok = mbar_wait<false>(smem_u32(&ctl.full[st]), (kc >> 1) & 1, abort, timeout_ns);
      if (!ok) break;
      tc_fence_after();
      const uint32_t base = smem_u32(smem + st * kStage);
#pragma unroll
      for (int kk = 0; kk < kGK / 16; ++kk) {
        const uint64_t ad = smem_desc(base + kk * 32, 16, 1024, kSwizzle128B);                  // K-major rows
        const uint64_t bd = smem_desc(base + kAChunk + kk * 2048, kBChunk, 1024, kSwizzle128B);  // N-major
        mma_ss(tmem, ad, bd, idesc, (kc | kk) ? 1u : 0u);
      }
      mma_commit(smem_u32(&ctl.empty[st]));
      if (kc + 2 < nk) {   // refill this stage once its MMAs have read it
        ok = mbar_wait<false>(smem_u32(&ctl.empty[st]), (kc >> 1) & 1, abort, timeout_ns);
        if (ok) load(kc + 2);
      }
    }
    mma_commit(smem_u32(&ctl.done));
    int dummy = 0;
    if (!mbar_wait<false>(smem_u32(&ctl.done), 0, &dummy, drain_ns)) ok = false;
    // loads still in flight land before the CTA may exit
    for (int kc = (nk > 2 ? nk - 2 : 0); kc < nk; ++kc)
      mbar_wait<false>(smem_u32(&ctl.full[kc & 1]), (kc >> 1) & 1, &dummy, drain_ns);
    if (!ok) {
      set_status(a.status, MLA_ERR_TIMEOUT);
      ctl.abort = 1;
    }
  }
  // epilogue: every warp waits for the accumulator, reads its 32 rows back
  {
    int dummy = 0;
    ok = __all_sync(0xffffffffu, mbar_wait<false>(smem_u32(&ctl.done), 0, &dummy, timeout_ns));
  }
  tc_fence_after();
  const int m = m0 + warp * 32 + lane;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
#pragma unroll 1
  for (int c = 0; c < kNT / 16 && ok; ++c) {
    uint32_t v[16];
    tmem_ld16(tmem + lane_off + 16 * c, v);
    tmem_wait_ld();
    if (m >= a.rows || ctl.abort) continue;
    uint32_t pk[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) pk[i] = pack2_bf16(__uint_as_float(v[2 * i]), __uint_as_float(v[2 * i + 1]));
    const uint4 o0 = make_uint4(pk[0], pk[1], pk[2], pk[3]), o1 = make_uint4(pk[4], pk[5], pk[6], pk[7]);
    uint4* dst = reinterpret_cast<uint4*>((uint16_t*)a.y + ((size_t)m * a.heads + h) * a.n + n0 + 16 * c);
    dst[0] = o0;
    dst[1] = o1;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kNT < 32 ? 32 : kNT);
  }
}

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

bool map3(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2, uint64_t s1, uint64_t s2,
          uint32_t b0, uint32_t b1, uint32_t b2) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {d0, d1, d2};
  const cuuint64_t strides[2] = {s1, s2};
  const cuuint32_t box[3] = {b0, b1, b2};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int kNT>
cudaError_t launch_nt(const GemmArgs& a, cudaStream_t s) {
  CUtensorMap tx, tw;
  // x [rows][heads][k]: box 64 k x 1 head x 128 rows (rows past the end read as zeros)
  if (!map3(&tx, a.x, a.k, a.heads, a.rows, (uint64_t)a.k * 2, (uint64_t)a.heads * a.k * 2, kGK, 1, kGM))
    return cudaErrorInvalidValue;
  // w [heads][k][n]: box 64 n x 64 k x 1 head
  if (!map3(&tw, a.w, a.n, a.k, a.heads, (uint64_t)a.n * 2, (uint64_t)a.k * a.n * 2, 64, kGK, 1))
    return cudaErrorInvalidValue;
  constexpr uint32_t kStage = kAChunk + (kNT / 64) * kBChunk;
  constexpr uint32_t smem = 2 * kStage + 1024 + 1024;
  static std::once_flag attr_once[64];
  int dev = 0;
  cudaGetDevice(&dev);
  cudaError_t err = cudaSuccess;
  std::call_once(attr_once[dev & 63], [&] {
    err = cudaFuncSetAttribute(head_gemm_kernel<kNT>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  });
  if (err != cudaSuccess) return err;
  const dim3 grid(a.n / kNT, a.heads, (a.rows + kGM - 1) / kGM);
  head_gemm_kernel<kNT><<<grid, 128, smem, s>>>(tx, tw, a, wait_timeout_ns(), drain_timeout_ns());
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_head_gemm(const GemmArgs& a, cudaStream_t s) {
  if (a.rows == 0) return cudaSuccess;
  if (a.n % 256 == 0) return launch_nt<256>(a, s);
  if (a.n % 128 == 0) return launch_nt<128>(a, s);
  return launch_nt<64>(a, s);
}

}  // namespace mla
