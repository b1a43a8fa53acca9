// Device helpers shared by the decode, combine and probe kernels: storage decoders,
// the sticky status word and the split plan.
#pragma once

#include <cstdint>

#include "mla_internal.h"
#include "../../include/mla_decode.h"

namespace mla {

__device__ __forceinline__ void set_status(int* status, int code) {
  if (*((volatile int*)status) == 0) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float((uint32_t)b << 16);
}

// OCP FP8 e4m3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinities,
// S.1111.111 = NaN) to fp32, written from that definition. Every code is exact in fp32.
__device__ __forceinline__ float e4m3_to_float(uint32_t code) {
  const uint32_t e = (code >> 3) & 0xF, m = code & 0x7;
  float v;
  if (e == 0)
    v = (float)m * 0x1p-9f;                                    // subnormal: m/8 * 2^-6
  else if (e == 0xF && m == 0x7)
    v = __uint_as_float(0x7FC00000u);                          // NaN
  else
    v = __uint_as_float(((e + 120u) << 23) | (m << 20));       // (1 + m/8) * 2^(e-7)
  return (code & 0x80) ? -v : v;
}

__device__ __forceinline__ float load_q(const void* p, int dtype, size_t i) {
  return dtype == kF32 ? __ldg((const float*)p + i) : bf16_bits_to_float(__ldg((const uint16_t*)p + i));
}

// ---------------------------------------------------------------------------- plan
//
// The work of one call is the batch-ordered list of every sequence's cache blocks
// ("tiles"): T = sum_b ceil(L_b / bs). With W' = min(W, T) active workers, worker
// w < W' owns tiles [floor(w T / W'), floor((w + 1) T / W')): at least one tile each,
// so the workers that touch a sequence are consecutive. The part of sequence b that
// worker w owns is one split; the splits of b are numbered from the first worker that
// touches b, and the split's partial result goes to workspace slot w + b.

__device__ __forceinline__ int clamp_len(int L, int cap, int* status) {
  if (L < 0 || L > cap) {
    set_status(status, MLA_ERR_BAD_SEQ_LEN);
    return L < 0 ? 0 : cap;
  }
  return L;
}

__device__ __forceinline__ int tiles_of(int Lc, int bs) { return (Lc + bs - 1) / bs; }

// Worker containing flat tile x (largest w with floor(w T / W) <= x).
__device__ __forceinline__ int worker_of_tile(long long x, long long T, int W) {
  return (int)(((x + 1) * (long long)W - 1) / T);
}

struct WorkerPlan {
  long long T;      // total tiles
  int W;            // active workers, min(W, T)
  long long start;  // first tile of this worker
  long long end;    // one past its last tile
  long long P0;     // flat index of sequence b0's first tile
  int b0;           // first sequence with a tile in [start, end)
};

// Executed by one full warp; every lane returns the same plan.
__device__ __forceinline__ WorkerPlan warp_plan(const int32_t* __restrict__ seq_lens, int B, int bs,
                                                int cap, int W, int w, int* status) {
  const int lane = threadIdx.x & 31;
  long long T = 0;
  for (int b = lane; b < B; b += 32) T += tiles_of(clamp_len(__ldg(seq_lens + b), cap, status), bs);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) T += __shfl_xor_sync(0xffffffffu, T, o);
  WorkerPlan p;
  p.T = T;
  p.W = (T > 0 && T < W) ? (int)T : W;
  p.start = (T > 0 && w < p.W) ? (long long)w * T / p.W : T;
  p.end = (T > 0 && w < p.W) ? (long long)(w + 1) * T / p.W : T;
  p.b0 = B;
  p.P0 = T;
  if (p.start >= p.end) return p;
  long long carry = 0;
  for (int base = 0; base < B; base += 32) {
    const int b = base + lane;
    const int n = b < B ? tiles_of(clamp_len(__ldg(seq_lens + b), cap, status), bs) : 0;
    long long incl = n;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      long long v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    const long long P = carry + incl - n;
    const bool hit = n > 0 && P <= p.start && p.start < P + n;
    const unsigned m = __ballot_sync(0xffffffffu, hit);
    if (m) {
      const int src = __ffs(m) - 1;
      p.b0 = base + src;
      p.P0 = __shfl_sync(0xffffffffu, P, src);
      return p;
    }
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  return p;
}

// One split of a sequence as seen by its worker.
struct Segment {
  int b;
  int tile_begin, tile_end;   // local tile range within sequence b
  int first_worker, splits;   // workers touching b
  int split;                  // this worker's index among them
  int Lc;                     // clamped sequence length
};

// Iterates the segments of a worker's range. Usage:
//   SegmentIter it(plan, ...); Segment sg; while (it.next(sg)) { ... }
struct SegmentIter {
  const int32_t* seq_lens;
  int B, bs, cap, W, w;
  int* status;
  WorkerPlan p;
  int b;
  long long P;

  __device__ SegmentIter(const WorkerPlan& plan, const int32_t* sl, int B_, int bs_, int cap_, int w_, int* st)
      : seq_lens(sl), B(B_), bs(bs_), cap(cap_), W(plan.W), w(w_), status(st), p(plan), b(plan.b0), P(plan.P0) {}

  __device__ bool next(Segment& sg) {
    while (b < B && P < p.end) {
      const int Lc = clamp_len(__ldg(seq_lens + b), cap, status);
      const int n = tiles_of(Lc, bs);
      const int cur = b++;
      const long long Pb = P;
      P += n;
      if (n == 0) continue;
      const long long s0 = Pb > p.start ? Pb : p.start;
      const long long s1 = (Pb + n) < p.end ? (Pb + n) : p.end;
      if (s1 <= s0) continue;
      sg.b = cur;
      sg.tile_begin = (int)(s0 - Pb);
      sg.tile_end = (int)(s1 - Pb);
      sg.first_worker = worker_of_tile(Pb, p.T, W);
      sg.splits = worker_of_tile(Pb + n - 1, p.T, W) - sg.first_worker + 1;
      sg.split = w - sg.first_worker;
      sg.Lc = Lc;
      return true;
    }
    return false;
  }
};

// Physical block of tile `tile` of sequence b, validated (bad ids read block 0).
__device__ __forceinline__ int checked_block(const int32_t* __restrict__ bt, int max_blocks, int b, int tile,
                                             int num_blocks, int* status) {
  int blk = __ldg(bt + (size_t)b * max_blocks + tile);
  if (blk < 0 || blk >= num_blocks) {
    set_status(status, MLA_ERR_BAD_BLOCK_ID);
    blk = 0;
  }
  return blk;
}

// Warp-collective: the part of sequence b in tiles [t0, t1) read something it may not: the
// sequence's length is out of range, a block id is out of range, or (sparse decode, sel_idx set)
// a listed position is outside the block table or maps to a bad block. Such rows are written as
// NaN.
__device__ __forceinline__ bool segment_poisoned(const DecodeArgs& a, int b, int t0, int t1) {
  const int lane = threadIdx.x & 31;
  const int L = __ldg(a.seq_lens + b);
  bool bad = L < 0 || L > a.len_cap;
  if (a.sel_idx == nullptr) {
    for (int t = t0 + lane; t < t1; t += 32) {
      const int blk = __ldg(a.block_table + (size_t)b * a.max_blocks + t);
      bad |= blk < 0 || blk >= a.num_blocks;
    }
  } else if (!bad) {
    const int pos_cap = a.max_blocks * a.bs;
    const int j1 = min(t1 * a.bs, L);
    for (int j = t0 * a.bs + lane; j < j1; j += 32) {
      const int t = __ldg(a.sel_idx + (size_t)b * a.top_k + j);
      const int blk = (t >= 0 && t < pos_cap) ? __ldg(a.block_table + (size_t)b * a.max_blocks + t / a.bs) : -1;
      bad |= blk < 0 || blk >= a.num_blocks;
    }
  }
  return __any_sync(0xffffffffu, bad);
}

}  // namespace mla
