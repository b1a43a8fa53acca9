// CUDA-core kernels: the fp32 SIMT decode (any latent width, any block size, every
// storage type), the log-sum-exp combine of split partials, and the plan probe.
//
// SIMT decode: CTA (worker w, row block) with one warp per query row (s, h) of the
// sequence being processed. The worker's cache blocks are streamed through shared
// memory in chunks of tokens decoded to fp32 (bf16 / e4m3 * scale / f32); every warp
// scores the chunk against its row's absorbed query with an fp32 online softmax in
// base 2 (score * scale * log2 e) and accumulates the latent rows as values.
#include <cfloat>
#include <cmath>

#include "mla_device.cuh"

namespace mla {
namespace {

constexpr int kWarps = 8;
constexpr int kThreads = kWarps * 32;
constexpr int kQV = kSimtMaxD / 32;   // per-lane query registers
constexpr int kAV = kSimtMaxR / 32;   // per-lane accumulator registers
constexpr int kChunkFloats = 12288;   // 48 KB of staged tokens

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ void store_out(void* out, int dtype, size_t i, float v) {
  if (dtype == kF32) {
    ((float*)out)[i] = v;
  } else {
    // round to nearest even bf16 (finite inputs; NaN stays NaN)
    uint32_t u = __float_as_uint(v);
    uint16_t h;
    if ((u & 0x7FFFFFFFu) > 0x7F800000u)
      h = 0x7FC0;
    else
      h = (uint16_t)((u + 0x7FFFu + ((u >> 16) & 1u)) >> 16);
    ((uint16_t*)out)[i] = h;
  }
}

__global__ void __launch_bounds__(kThreads) simt_decode_kernel(const DecodeArgs a, int chunk) {
  extern __shared__ float tok[];   // [chunk][D]
  __shared__ WorkerPlan s_plan;
  const int D = a.r + a.d_r;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int w = blockIdx.x;
  const int row = blockIdx.y * kWarps + warp;
  const bool row_ok = row < a.rows;
  const int s = row_ok ? row / a.H : 0;
  const int cap = a.len_cap;

  if (warp == 0) {
    WorkerPlan p = warp_plan(a.seq_lens, a.B, a.bs, cap, a.W, w, a.status);
    if (lane == 0) s_plan = p;
  }
  __syncthreads();
  const WorkerPlan plan = s_plan;

  SegmentIter it(plan, a.seq_lens, a.B, a.bs, cap, w, a.status);
  Segment sg;
  while (it.next(sg)) {
    const int b = sg.b;
    if (sg.split == 0 && blockIdx.y == 0 && threadIdx.x == 0) {
      a.meta[2 * b] = sg.first_worker;
      a.meta[2 * b + 1] = sg.splits;
    }
    // absorbed query of this row, lane-strided
    float q[kQV];
    const size_t qrow = (size_t)b * a.rows + row;
#pragma unroll
    for (int i = 0; i < kQV; ++i) {
      const int k = lane + 32 * i;
      float v = 0.f;
      if (row_ok && k < a.r) v = load_q(a.q_lat, a.q_dtype, qrow * a.r + k);
      else if (row_ok && k < D) v = load_q(a.q_rope, a.q_dtype, qrow * a.d_r + (k - a.r));
      q[i] = v;
    }
    float acc[kAV];
#pragma unroll
    for (int i = 0; i < kAV; ++i) acc[i] = 0.f;
    float m = -INFINITY, l = 0.f;

    const int t_begin = sg.tile_begin * a.bs;
    const int t_end = min(sg.tile_end * a.bs, sg.Lc);
    const int n_row = a.causal ? sg.Lc - a.Sq + 1 + s : sg.Lc;   // tokens this row may see
    const int hi = min(t_end, n_row);

    for (int c0 = t_begin; c0 < t_end; c0 += chunk) {
      const int cn = min(chunk, t_end - c0);
      __syncthreads();
      for (int j = 0; j < cn; ++j) {
        const int t = c0 + j;
        const int blk = checked_block(a.block_table, a.max_blocks, b, t / a.bs, a.num_blocks, a.status);
        const size_t slot = (size_t)blk * a.bs + (t % a.bs);
        for (int k = threadIdx.x; k < D; k += kThreads) {
          float v;
          if (a.cache_dtype == kE4M3) {
            if (k < a.r)
              v = e4m3_to_float(__ldg((const uint8_t*)a.cache + slot * a.r + k)) * __ldg(a.kv_scale + slot);
            else
              v = bf16_bits_to_float(__ldg(a.k_rope + slot * a.d_r + (k - a.r)));
          } else if (a.cache_dtype == kBF16) {
            v = bf16_bits_to_float(__ldg((const uint16_t*)a.cache + slot * D + k));
          } else {
            v = __ldg((const float*)a.cache + slot * D + k);
          }
          tok[j * D + k] = v;
        }
      }
      __syncthreads();
      if (!row_ok) continue;
      const int jn = min(cn, hi - c0);
      for (int j = 0; j < jn; ++j) {
        const float* c = tok + j * D;
        float d = 0.f;
#pragma unroll
        for (int i = 0; i < kQV; ++i) {
          const int k = lane + 32 * i;
          if (k < D) d = fmaf(q[i], c[k], d);
        }
        const float x = warp_sum(d) * a.scale_log2;
        const float m_new = fmaxf(m, x);
        const float corr = exp2f(m - m_new);
        const float p = exp2f(x - m_new);
        l = fmaf(l, corr, p);
#pragma unroll
        for (int i = 0; i < kAV; ++i) {
          const int k = lane + 32 * i;
          if (k < a.r) acc[i] = fmaf(acc[i], corr, p * c[k]);
        }
        m = m_new;
      }
    }
    const bool poisoned = segment_poisoned(a, b, sg.tile_begin, sg.tile_end);
    if (!row_ok) continue;
    const float qnan = __uint_as_float(0x7FC00000u);
    const float inv = poisoned ? qnan : l > 0.f ? 1.f / l : 0.f;
    const float lse_v = poisoned ? qnan : l > 0.f ? (m + log2f(l)) * 0.69314718055994531f : -INFINITY;
    if (sg.splits == 1) {
#pragma unroll
      for (int i = 0; i < kAV; ++i) {
        const int k = lane + 32 * i;
        if (k < a.r) store_out(a.out, a.out_dtype, qrow * a.r + k, acc[i] * inv);
      }
      if (lane == 0) a.lse[qrow] = lse_v;
    } else {
      const size_t prow = (size_t)(w + b) * a.rows + row;
#pragma unroll
      for (int i = 0; i < kAV; ++i) {
        const int k = lane + 32 * i;
        if (k < a.r) a.o_part[prow * a.r + k] = acc[i] * inv;
      }
      if (lane == 0) a.lse_part[prow] = lse_v;
    }
  }
}

// One warp per (b, row): merge the partials of split sequences, fill empty ones. The split of
// each sequence is recomputed here from seq_lens with the plan's formula (nothing read from the
// workspace is trusted for indexing). Rows of a sequence with a seq_len out of range, and rows
// whose partials carry a NaN log-sum-exp (a decode wait timed out, or a bad block id), are
// written as NaN.
__global__ void __launch_bounds__(kThreads) combine_kernel(const DecodeArgs a) {
  __shared__ long long s_sum[kWarps][2];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int b = blockIdx.x;
  const int cap = a.len_cap;
  // tiles before sequence b and in total, as the decode kernels' plan counts them
  long long before = 0, total = 0;
  for (int i = threadIdx.x; i < a.B; i += kThreads) {
    const int L = __ldg(a.seq_lens + i);
    const long long n = tiles_of(L < 0 ? 0 : (L > cap ? cap : L), a.bs);
    total += n;
    if (i < b) before += n;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    before += __shfl_xor_sync(0xffffffffu, before, o);
    total += __shfl_xor_sync(0xffffffffu, total, o);
  }
  if (lane == 0) {
    s_sum[warp][0] = before;
    s_sum[warp][1] = total;
  }
  __syncthreads();
  before = total = 0;
#pragma unroll
  for (int i = 0; i < kWarps; ++i) {
    before += s_sum[i][0];
    total += s_sum[i][1];
  }
  const int row = blockIdx.y * kWarps + warp;
  if (row >= a.rows) return;
  const size_t orow = (size_t)b * a.rows + row;
  const int raw = __ldg(a.seq_lens + b);
  const float qnan = __uint_as_float(0x7FC00000u);
  if (raw < 0 || raw > cap) {
    for (int k = lane; k < a.r; k += 32) store_out(a.out, a.out_dtype, orow * a.r + k, qnan);
    if (lane == 0) a.lse[orow] = qnan;
    return;
  }
  const long long n = tiles_of(raw, a.bs);
  if (n == 0) {
    for (int k = lane; k < a.r; k += 32) store_out(a.out, a.out_dtype, orow * a.r + k, 0.f);
    if (lane == 0) a.lse[orow] = -INFINITY;
    return;
  }
  const int Wa = (total < a.W) ? (int)total : a.W;
  const int first = worker_of_tile(before, total, Wa);
  const int splits = worker_of_tile(before + n - 1, total, Wa) - first + 1;
  if (splits <= 1) return;   // the decode wrote this row directly
  const size_t slot0 = (size_t)first + b;
  float M = -INFINITY;
  bool has_nan = false;
  for (int i = lane; i < splits; i += 32) {
    const float v = a.lse_part[(slot0 + i) * a.rows + row];
    has_nan |= v != v;
    M = fmaxf(M, v);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) M = fmaxf(M, __shfl_xor_sync(0xffffffffu, M, o));
  if (__any_sync(0xffffffffu, has_nan)) {
    for (int k = lane; k < a.r; k += 32) store_out(a.out, a.out_dtype, orow * a.r + k, qnan);
    if (lane == 0) a.lse[orow] = qnan;
    return;
  }
  if (M == -INFINITY) {
    for (int k = lane; k < a.r; k += 32) store_out(a.out, a.out_dtype, orow * a.r + k, 0.f);
    if (lane == 0) a.lse[orow] = -INFINITY;
    return;
  }
  float Z = 0.f;
  for (int i = lane; i < splits; i += 32) Z += expf(a.lse_part[(slot0 + i) * a.rows + row] - M);
  Z = warp_sum(Z);
  const float lse_v = M + logf(Z);
  if (a.r % 4 == 0) {
    // 512 channels per pass, 16 per lane as four float4 pieces; each split's pieces are
    // independent loads, so a split costs one memory latency, not one per piece. The split
    // weights come from lane i (splits <= 32) by shuffle; the output goes out 4 channels per store.
    const float wl = lane < splits ? expf(a.lse_part[(slot0 + lane) * a.rows + row] - lse_v) : 0.f;
    // 4 output channels per store when the output allows it (the SIMT path takes 4-byte
    // aligned outputs)
    const bool vec_out = ((uintptr_t)a.out % (a.out_dtype == kF32 ? 16u : 8u)) == 0;
    for (int k0 = 0; k0 < a.r; k0 += 512) {
      float4 o[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) o[u] = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 2
      for (int i = 0; i < splits; ++i) {
        const size_t prow = (slot0 + i) * a.rows + row;
        const float wgt = i < 32 ? __shfl_sync(0xffffffffu, wl, i) : expf(a.lse_part[prow] - lse_v);
        if (wgt == 0.f) continue;
        const float* src = a.o_part + prow * a.r;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int k = k0 + 4 * lane + 128 * u;
          if (k < a.r) {
            const float4 v = *reinterpret_cast<const float4*>(src + k);
            o[u].x = fmaf(wgt, v.x, o[u].x);
            o[u].y = fmaf(wgt, v.y, o[u].y);
            o[u].z = fmaf(wgt, v.z, o[u].z);
            o[u].w = fmaf(wgt, v.w, o[u].w);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int k = k0 + 4 * lane + 128 * u;
        if (k < a.r && !vec_out) {
          const size_t e = orow * a.r + k;
          store_out(a.out, a.out_dtype, e, o[u].x);
          store_out(a.out, a.out_dtype, e + 1, o[u].y);
          store_out(a.out, a.out_dtype, e + 2, o[u].z);
          store_out(a.out, a.out_dtype, e + 3, o[u].w);
        } else if (k < a.r) {
          const size_t e = orow * a.r + k;
          if (a.out_dtype == kF32) {
            *reinterpret_cast<float4*>((float*)a.out + e) = o[u];
          } else {
            uint32_t lo, hi;   // round to nearest even; NaN stays NaN
            asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(lo) : "f"(o[u].y), "f"(o[u].x));
            asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(hi) : "f"(o[u].w), "f"(o[u].z));
            *reinterpret_cast<uint2*>((uint16_t*)a.out + e) = make_uint2(lo, hi);
          }
        }
      }
    }
  } else {
    for (int k0 = 0; k0 < a.r; k0 += 32 * 4) {
      float o[4] = {0.f, 0.f, 0.f, 0.f};
      for (int i = 0; i < splits; ++i) {
        const size_t prow = (slot0 + i) * a.rows + row;
        const float wgt = expf(a.lse_part[prow] - lse_v);
        if (wgt == 0.f) continue;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int k = k0 + lane + 32 * u;
          if (k < a.r) o[u] = fmaf(wgt, a.o_part[prow * a.r + k], o[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int k = k0 + lane + 32 * u;
        if (k < a.r) store_out(a.out, a.out_dtype, orow * a.r + k, o[u]);
      }
    }
  }
  if (lane == 0) a.lse[orow] = lse_v;
}

__global__ void __launch_bounds__(32) plan_probe_kernel(const DecodeArgs a, int32_t* token_slot,
                                                         int32_t* token_worker) {
  const int w = blockIdx.x, lane = threadIdx.x;
  const int cap = a.len_cap;
  const WorkerPlan p = warp_plan(a.seq_lens, a.B, a.bs, cap, a.W, w, a.status);
  SegmentIter it(p, a.seq_lens, a.B, a.bs, cap, w, a.status);
  Segment sg;
  while (it.next(sg)) {
    if (sg.split == 0 && lane == 0) {
      a.meta[2 * sg.b] = sg.first_worker;
      a.meta[2 * sg.b + 1] = sg.splits;
    }
    const int t1 = min(sg.tile_end * a.bs, sg.Lc);
    for (int t = sg.tile_begin * a.bs + lane; t < t1; t += 32) {
      const int blk = checked_block(a.block_table, a.max_blocks, sg.b, t / a.bs, a.num_blocks, a.status);
      const size_t o = (size_t)sg.b * a.max_blocks * a.bs + t;
      token_slot[o] = blk * a.bs + t % a.bs;
      token_worker[o] = w;
    }
  }
}

}  // namespace

cudaError_t launch_simt_decode(const DecodeArgs& a, cudaStream_t s) {
  const int D = a.r + a.d_r;
  int chunk = kChunkFloats / D;
  if (chunk > 32) chunk = 32;
  if (chunk < 1) chunk = 1;
  dim3 grid(a.W, (a.rows + kWarps - 1) / kWarps);
  simt_decode_kernel<<<grid, kThreads, sizeof(float) * chunk * D, s>>>(a, chunk);
  return cudaGetLastError();
}

cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t s) {
  dim3 grid(a.B, (a.rows + kWarps - 1) / kWarps);
  combine_kernel<<<grid, kThreads, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_plan_probe(const DecodeArgs& a, int32_t* token_slot, int32_t* token_worker,
                              cudaStream_t s) {
  plan_probe_kernel<<<a.W, 32, 0, s>>>(a, token_slot, token_worker);
  return cudaGetLastError();
}

}  // namespace mla
