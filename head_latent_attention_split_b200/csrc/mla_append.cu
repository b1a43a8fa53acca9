// Paged cache append: the latent and RoPE key of each sequence's new tokens written into
// the slots mla_decode reads, with optional e4m3 per-token quantisation and RoPE
// rotation. See mla_cache_append in include/mla_decode.h.
//
// One warp per new token; the latent is moved lane-strided (coalesced), the per-token
// scale is a warp max reduction. The e4m3 codes come from the hardware fp32 -> e4m3x2
// conversion (round to nearest even, saturated), applied to the IEEE fp32 quotient
// c / scale. The RoPE angle pos * theta_i and the rotation are computed in fp64 and the
// result is rounded to fp32, then to the cache type.
#include <cuda_bf16.h>

#include "mla_device.cuh"

namespace mla {
namespace {

__device__ __forceinline__ float load_in(const void* p, int dtype, size_t i) {
  return dtype == kF32 ? ((const float*)p)[i] : bf16_bits_to_float(((const uint16_t*)p)[i]);
}

// fp32 -> bf16 bits, round to nearest even (finite inputs)
__device__ __forceinline__ uint16_t f32_to_bf16_bits(float x) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(x));
}

// two fp32 -> e4m3 codes (lo in the low byte), round to nearest even, saturated to +-448
__device__ __forceinline__ uint16_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

__global__ void __launch_bounds__(256) append_kernel(const AppendArgs a) {
  const int lane = threadIdx.x & 31;
  const long long tok = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (tok >= (long long)a.B * a.Sq) return;
  const int b = (int)(tok / a.Sq), s = (int)(tok % a.Sq);
  const long long pos = (long long)__ldg(a.seq_lens + b) - a.Sq + s;
  if (pos < 0 || pos >= (long long)a.max_blocks * a.bs) {
    if (lane == 0) set_status(a.status, MLA_ERR_BAD_SEQ_LEN);
    return;
  }
  const int blk = __ldg(a.block_table + (size_t)b * a.max_blocks + pos / a.bs);
  if (blk < 0 || blk >= a.num_blocks) {
    if (lane == 0) set_status(a.status, MLA_ERR_BAD_BLOCK_ID);
    return;
  }
  const size_t slot = (size_t)blk * a.bs + (size_t)(pos % a.bs);
  const size_t src = (size_t)tok;   // row of c_new / k_rope_new
  const int D = a.r + a.d_r;

  // ---- latent
  if (a.cache_dtype == kE4M3) {
    const uint16_t* c = (const uint16_t*)a.c_new + src * a.r;
    float amax = 0.f;
    for (int k = lane; k < a.r; k += 32) amax = fmaxf(amax, fabsf(bf16_bits_to_float(c[k])));
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
    const float scale = __fdiv_rn(amax, 448.f);
    uint16_t* codes = (uint16_t*)((uint8_t*)a.cache + slot * a.r);   // r is even
    for (int k2 = lane; k2 < a.r / 2; k2 += 32) {
      const float v0 = bf16_bits_to_float(c[2 * k2]), v1 = bf16_bits_to_float(c[2 * k2 + 1]);
      const float q0 = scale > 0.f ? __fdiv_rn(v0, scale) : 0.f;
      const float q1 = scale > 0.f ? __fdiv_rn(v1, scale) : 0.f;
      codes[k2] = f32x2_to_e4m3x2(q0, q1);
    }
    if (lane == 0) a.kv_scale[slot] = scale;
  } else if (a.cache_dtype == kBF16) {
    const uint16_t* c = (const uint16_t*)a.c_new + src * a.r;
    uint16_t* dst = (uint16_t*)a.cache + slot * D;
    for (int k = lane; k < a.r; k += 32) dst[k] = c[k];
  } else {
    const float* c = (const float*)a.c_new + src * a.r;
    float* dst = (float*)a.cache + slot * D;
    for (int k = lane; k < a.r; k += 32) dst[k] = c[k];
  }

  // ---- RoPE key (rotated at pos when asked)
  const int npairs = a.rope ? a.d_r / 2 : 0;
  for (int i = lane; i < npairs; i += 32) {
    const float x0 = load_in(a.k_new, a.in_dtype, src * a.d_r + 2 * i);
    const float x1 = load_in(a.k_new, a.in_dtype, src * a.d_r + 2 * i + 1);
    const double theta = pow((double)a.rope_base, -2.0 * (double)i / (double)a.d_r);
    double sn, cs;
    sincos((double)pos * theta, &sn, &cs);
    const float y0 = (float)((double)x0 * cs - (double)x1 * sn);
    const float y1 = (float)((double)x0 * sn + (double)x1 * cs);
    if (a.cache_dtype == kF32) {
      float* dst = (float*)a.cache + slot * D + a.r;
      dst[2 * i] = y0;
      dst[2 * i + 1] = y1;
    } else {
      uint16_t* dst = a.cache_dtype == kE4M3 ? a.k_rope + slot * a.d_r : (uint16_t*)a.cache + slot * D + a.r;
      dst[2 * i] = f32_to_bf16_bits(y0);
      dst[2 * i + 1] = f32_to_bf16_bits(y1);
    }
  }
  if (!a.rope) {
    for (int j = lane; j < a.d_r; j += 32) {
      if (a.cache_dtype == kF32) {
        ((float*)a.cache)[slot * D + a.r + j] = ((const float*)a.k_new)[src * a.d_r + j];
      } else {
        uint16_t* dst = a.cache_dtype == kE4M3 ? a.k_rope + slot * a.d_r : (uint16_t*)a.cache + slot * D + a.r;
        dst[j] = ((const uint16_t*)a.k_new)[src * a.d_r + j];
      }
    }
  }
}

}  // namespace

cudaError_t launch_cache_append(const AppendArgs& a, cudaStream_t s) {
  const long long warps = (long long)a.B * a.Sq;
  if (warps == 0) return cudaSuccess;
  const unsigned grid = (unsigned)((warps + 7) / 8);
  append_kernel<<<grid, 256, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace mla
