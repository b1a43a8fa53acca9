// Internal interface between the C-ABI host layer (mla_api.cu) and the kernel
// translation units. Not installed; the public interface is include/mla_decode.h.
#pragma once

#include <cstddef>
#include <cstdint>

#include <cuda_runtime.h>

namespace mla {

enum : int { kF32 = 0, kBF16 = 1, kE4M3 = 2 };

// Everything a decode / combine / probe kernel needs, by value.
struct DecodeArgs {
  int B, Sq, H, r, d_r;
  int bs;              // block_size (tokens per cache block)
  int num_blocks;
  int max_blocks;      // block_table row stride
  int q_dtype, cache_dtype, out_dtype;
  int causal;
  int rows;            // Sq * H query rows per sequence
  int len_cap;         // largest valid seq_lens entry: max_blocks * bs (sparse decode: also <= top_k)
  int W;               // workers sharing the flat block list
  float scale;         // softmax scale
  float scale_log2;    // softmax scale * log2(e)
  const void* q_lat;
  const void* q_rope;
  const void* cache;           // F32/BF16: [nb, bs, r + d_r]; E4M3: codes [nb, bs, r]
  const uint16_t* k_rope;      // E4M3 only: bf16 [nb, bs, d_r]
  const float* kv_scale;       // E4M3 only: [nb, bs]
  const int32_t* block_table;  // [B, max_blocks]
  const int32_t* seq_lens;     // [B]; sparse decode: the selected token counts
  const int32_t* sel_idx;      // sparse decode only: [B, top_k] selected positions, else null
  int top_k;                   // sparse decode only: row stride of sel_idx
  void* out;                   // [B, Sq, H, r] out_dtype
  float* lse;                  // [B, Sq, H]
  // workspace
  int32_t* meta;               // [B, 2]: first worker, number of splits
  float* lse_part;             // [slots, rows]
  float* o_part;               // [slots, rows, r] (normalised partial outputs)
  int* status;                 // sticky device status word
};

// Workspace regions; every offset is 256-byte aligned.
struct WorkspaceLayout {
  size_t meta_off, lse_off, o_off, total;
  int64_t slots;
};

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Limit, in nanoseconds, of the bounded waits on a kernel's pipeline (default 2 s; set with
// mla_set_wait_timeout_ns). A wait that runs out sets MLA_ERR_TIMEOUT.
uint64_t wait_timeout_ns();
// Limit of the waits that let a CTA's in-flight copies and MMAs land before it exits; never
// shorter than the pipeline limit, so work already issued always completes.
constexpr uint64_t kDrainTimeoutNs = 2000000000ull;
inline uint64_t drain_timeout_ns() {
  const uint64_t t = wait_timeout_ns();
  return t > kDrainTimeoutNs ? t : kDrainTimeoutNs;
}

inline WorkspaceLayout workspace_layout(int B, int W, int rows, int r) {
  WorkspaceLayout L;
  // worker w's part of sequence b uses slot w + b (unique: workers own increasing,
  // contiguous block ranges of the batch-ordered block list)
  L.slots = (B > 0 && W > 0) ? (int64_t)W + B - 1 : 0;
  L.meta_off = 0;
  L.lse_off = align_up(sizeof(int32_t) * 2 * (size_t)B, 256);
  L.o_off = L.lse_off + align_up(sizeof(float) * (size_t)L.slots * rows, 256);
  L.total = L.o_off + align_up(sizeof(float) * (size_t)L.slots * rows * r, 256);
  return L;
}

// SIMT (CUDA-core, fp32) decode: any r <= kSimtMaxR, r + d_r <= kSimtMaxD.
constexpr int kSimtMaxR = 1024;
constexpr int kSimtMaxD = 1280;
cudaError_t launch_simt_decode(const DecodeArgs& a, cudaStream_t s);

// Log-sum-exp merge of split partials (and the fill of empty sequences).
cudaError_t launch_combine(const DecodeArgs& a, cudaStream_t s);

// Plan probe for tests.
cudaError_t launch_plan_probe(const DecodeArgs& a, int32_t* token_slot, int32_t* token_worker,
                              cudaStream_t s);

// Arguments of the paged cache append kernel (mla_append.cu).
struct AppendArgs {
  int B, Sq, r, d_r, bs, num_blocks, max_blocks;
  int in_dtype, cache_dtype, rope;
  float rope_base;
  const void* c_new;           // [B, Sq, r] in_dtype
  const void* k_new;           // [B, Sq, d_r] in_dtype
  void* cache;                 // F32/BF16: [nb, bs, r + d_r]; E4M3: codes [nb, bs, r]
  uint16_t* k_rope;            // E4M3 only: bf16 [nb, bs, d_r]
  float* kv_scale;             // E4M3 only: [nb, bs]
  const int32_t* block_table;  // [B, max_blocks]
  const int32_t* seq_lens;     // [B]
  int* status;
};
cudaError_t launch_cache_append(const AppendArgs& a, cudaStream_t s);

// Arguments of the per-head GEMM (mla_gemm.cu): y[m, h, :] = x[m, h, :] . w[h].
struct GemmArgs {
  int rows, heads, k, n;   // k, n multiples of 64
  const void* x;           // [rows, heads, k] bf16
  const void* w;           // [heads, k, n] bf16
  void* y;                 // [rows, heads, n] bf16
  int* status;
};
cudaError_t launch_head_gemm(const GemmArgs& a, cudaStream_t s);

// Sparse attention side kernels (mla_dsa.cu): the FP8 lightning indexer and top-k.
constexpr int kDsaHeads = 64;    // indexer heads H^I of the tensor path
constexpr int kDsaDim = 128;     // indexer width d^I of the tensor path
struct DsaArgs {
  int B, Sq, bs, num_blocks, max_blocks, max_seq_len, top_k, causal;
  const uint8_t* q;            // [B, Sq, 64, 128] e4m3
  const float* q_scale;        // [B, Sq, 64]
  const float* w;              // [B, Sq, 64]
  const uint8_t* k;            // [num_blocks, bs, 128] e4m3
  const float* k_scale;        // [num_blocks, bs]
  const int32_t* block_table;  // [B, max_blocks]
  const int32_t* seq_lens;     // [B]
  float* scores;               // [B, Sq, max_seq_len]
  int32_t* indices;            // [B, Sq, top_k]
  int32_t* counts;             // [B, Sq]
  int* status;
};
cudaError_t launch_dsa_index(const DsaArgs& a, cudaStream_t s);
cudaError_t launch_dsa_topk(const DsaArgs& a, cudaStream_t s);

}  // namespace mla
