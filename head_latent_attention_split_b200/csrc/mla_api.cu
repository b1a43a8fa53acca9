// C-ABI host layer of libmla_decode.so: argument validation, kernel choice, workspace
// layout, launches, the sticky device status word. See include/mla_decode.h.
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>

#include "../../include/mla_decode.h"
#include "mla_internal.h"
#include "mla_tc.h"

namespace {

__device__ int g_mla_status;   // sticky per-device status word (first error wins)

std::atomic<uint64_t> g_wait_timeout_ns{mla::kDrainTimeoutNs};

constexpr int kMaxDevices = 64;
int* g_status_ptr[kMaxDevices];
std::once_flag g_status_once[kMaxDevices];

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return -1;
  return dev;
}

int* status_word(int dev) {
  if (dev < 0 || dev >= kMaxDevices) return nullptr;
  std::call_once(g_status_once[dev], [dev] {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_mla_status) == cudaSuccess) g_status_ptr[dev] = (int*)p;
  });
  return g_status_ptr[dev];
}

int sm_count() {
  int dev = current_device();
  if (dev < 0) return -1;
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return -1;
  return n;
}

bool dtype_ok(int d) { return d == MLA_DTYPE_F32 || d == MLA_DTYPE_BF16 || d == MLA_DTYPE_E4M3; }

size_t elem_size(int d) { return d == MLA_DTYPE_F32 ? 4 : d == MLA_DTYPE_BF16 ? 2 : 1; }

mla_status_t check_shape(const mla_decode_params_t* p) {
  if (!p) return MLA_ERR_INVALID_ARG;
  if (p->batch < 0 || p->q_len < 1 || p->num_heads < 1 || p->kv_rank < 1 || p->rope_dim < 0 ||
      p->block_size < 1 || p->num_blocks < 0 || p->max_blocks_per_seq < 1 || p->num_workers < 0 ||
      p->reserved != 0)
    return MLA_ERR_INVALID_ARG;
  if (p->batch > 0 && p->num_blocks < 1) return MLA_ERR_INVALID_ARG;
  if (!dtype_ok(p->q_dtype) || !dtype_ok(p->cache_dtype) || !dtype_ok(p->out_dtype))
    return MLA_ERR_INVALID_ARG;
  const bool triple_ok =
      (p->q_dtype == MLA_DTYPE_F32 && p->cache_dtype == MLA_DTYPE_F32 && p->out_dtype == MLA_DTYPE_F32) ||
      (p->q_dtype == MLA_DTYPE_BF16 && (p->cache_dtype == MLA_DTYPE_BF16 || p->cache_dtype == MLA_DTYPE_E4M3) &&
       (p->out_dtype == MLA_DTYPE_BF16 || p->out_dtype == MLA_DTYPE_F32));
  if (!triple_ok) return MLA_ERR_INVALID_ARG;
  if (!std::isfinite(p->softmax_scale)) return MLA_ERR_INVALID_ARG;
  if (p->causal != 0 && p->causal != 1) return MLA_ERR_INVALID_ARG;
  if (p->kernel < MLA_KERNEL_AUTO || p->kernel > MLA_KERNEL_TC_PAIR) return MLA_ERR_INVALID_ARG;
  // 32-bit token and slot indices inside the kernels
  if ((int64_t)p->max_blocks_per_seq * p->block_size > (1ll << 30)) return MLA_ERR_UNSUPPORTED;
  if ((int64_t)p->num_blocks * p->block_size > (1ll << 31) - 1) return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

bool simt_ok(const mla_decode_params_t* p) {
  return p->kv_rank <= mla::kSimtMaxR && p->kv_rank + p->rope_dim <= mla::kSimtMaxD;
}

// Resolve the kernel and the worker count. needs_device: the SM count was required.
// sparse: the call is a sparse decode. AUTO then keeps the single-CTA tensor-core kernel: its
// row gathers per tile are fewer than the split-role kernel's (which fetches each row for both
// CTAs), and gathers bound both (measured 0.116 vs 0.158 ms for the 128K / k = 2048 step).
mla_status_t resolve(const mla_decode_params_t* p, int* kernel, int* workers, bool sparse = false) {
  mla_status_t st = check_shape(p);
  if (st) return st;
  const bool tc_ok = mla::tc_supported(p->kv_rank, p->rope_dim, p->block_size, p->q_dtype, p->cache_dtype,
                                       p->out_dtype, p->q_len * p->num_heads);
  int k = p->kernel;
  if (k == MLA_KERNEL_AUTO) {
    if (!tc_ok || !mla::kTcAuto)
      k = MLA_KERNEL_SIMT;
    else
      k = (!sparse && p->cache_dtype == MLA_DTYPE_BF16) ? MLA_KERNEL_TC_PAIR : MLA_KERNEL_TCGEN05;
  }
  if (k == MLA_KERNEL_TCGEN05 && !tc_ok) return MLA_ERR_UNSUPPORTED;
  if (k == MLA_KERNEL_TC_PAIR && (!tc_ok || p->cache_dtype != MLA_DTYPE_BF16)) return MLA_ERR_UNSUPPORTED;
  if (k == MLA_KERNEL_SIMT && !simt_ok(p)) return MLA_ERR_UNSUPPORTED;
  int W = p->num_workers;
  if (W == 0) {
    const int sms = sm_count();
    if (sms <= 0) return MLA_ERR_CUDA;
    if (k == MLA_KERNEL_TCGEN05 || k == MLA_KERNEL_TC_PAIR) {
      W = mla::tc_auto_workers(sms, p->q_len * p->num_heads);
    } else {
      const int row_blocks = (p->q_len * p->num_heads + 7) / 8;
      W = 4 * sms / row_blocks;
    }
    if (W < 1) W = 1;
  }
  if ((k == MLA_KERNEL_TCGEN05 || k == MLA_KERNEL_TC_PAIR) && !mla::tc_workers_ok(W, p->q_len * p->num_heads)) return MLA_ERR_UNSUPPORTED;
  if (W > 65535 * 8) return MLA_ERR_UNSUPPORTED;
  *kernel = k;
  *workers = W;
  return MLA_OK;
}

mla::WorkspaceLayout layout_for(const mla_decode_params_t* p, int W) {
  return mla::workspace_layout(p->batch, W, p->q_len * p->num_heads, p->kv_rank);
}

bool aligned(const void* ptr, size_t a) { return ((uintptr_t)ptr % a) == 0; }

mla::DecodeArgs make_args(const mla_decode_params_t* p, int W) {
  mla::DecodeArgs a{};
  a.B = p->batch;
  a.Sq = p->q_len;
  a.H = p->num_heads;
  a.r = p->kv_rank;
  a.d_r = p->rope_dim;
  a.bs = p->block_size;
  a.num_blocks = p->num_blocks;
  a.max_blocks = p->max_blocks_per_seq;
  a.q_dtype = p->q_dtype;
  a.cache_dtype = p->cache_dtype;
  a.out_dtype = p->out_dtype;
  a.causal = p->causal;
  a.rows = p->q_len * p->num_heads;
  a.len_cap = p->max_blocks_per_seq * p->block_size;
  a.W = W;
  a.scale = p->softmax_scale;
  a.scale_log2 = (float)((double)p->softmax_scale * 1.4426950408889634);
  return a;
}

}  // namespace

uint64_t mla::wait_timeout_ns() { return g_wait_timeout_ns.load(std::memory_order_relaxed); }

extern "C" {

int32_t mla_abi_version(void) { return MLA_DECODE_ABI_VERSION; }

mla_status_t mla_set_wait_timeout_ns(uint64_t ns) {
  g_wait_timeout_ns.store(ns ? ns : mla::kDrainTimeoutNs, std::memory_order_relaxed);
  return MLA_OK;
}

uint64_t mla_get_wait_timeout_ns(void) { return mla::wait_timeout_ns(); }

const char* mla_status_string(int32_t s) {
  switch (s) {
    case MLA_OK: return "MLA_OK";
    case MLA_ERR_INVALID_ARG: return "MLA_ERR_INVALID_ARG";
    case MLA_ERR_UNSUPPORTED: return "MLA_ERR_UNSUPPORTED";
    case MLA_ERR_ALIGNMENT: return "MLA_ERR_ALIGNMENT";
    case MLA_ERR_WORKSPACE_TOO_SMALL: return "MLA_ERR_WORKSPACE_TOO_SMALL";
    case MLA_ERR_CUDA: return "MLA_ERR_CUDA";
    case MLA_ERR_BAD_BLOCK_ID: return "MLA_ERR_BAD_BLOCK_ID";
    case MLA_ERR_BAD_SEQ_LEN: return "MLA_ERR_BAD_SEQ_LEN";
    case MLA_ERR_TIMEOUT: return "MLA_ERR_TIMEOUT";
    default: return "MLA_ERR_UNKNOWN";
  }
}

mla_status_t mla_decode_resolve(const mla_decode_params_t* p, int32_t* kernel, int32_t* num_workers) {
  if (!kernel || !num_workers) return MLA_ERR_INVALID_ARG;
  int k = 0, W = 0;
  mla_status_t st = resolve(p, &k, &W);
  if (st) return st;
  *kernel = k;
  *num_workers = W;
  return MLA_OK;
}

mla_status_t mla_decode_workspace_size(const mla_decode_params_t* p, size_t* bytes) {
  if (!bytes) return MLA_ERR_INVALID_ARG;
  int k = 0, W = 0;
  mla_status_t st = resolve(p, &k, &W);
  if (st) return st;
  *bytes = layout_for(p, W).total;
  return MLA_OK;
}

namespace {
mla_status_t decode_impl(const mla_decode_params_t* p, const void* q_lat, const void* q_rope,
                         const void* kv_cache, const void* k_rope_cache, const float* kv_scale,
                         const int32_t* block_table, const int32_t* seq_lens, void* out, float* lse,
                         void* workspace, size_t workspace_bytes, void* stream, void* const* events) {
  int kernel = 0, W = 0;
  mla_status_t st = resolve(p, &kernel, &W);
  if (st) return st;
  if (p->batch == 0) return MLA_OK;
  if (!q_lat || !kv_cache || !block_table || !seq_lens || !out || !lse) return MLA_ERR_INVALID_ARG;
  if (p->rope_dim > 0 && !q_rope) return MLA_ERR_INVALID_ARG;
  if (p->cache_dtype == MLA_DTYPE_E4M3) {
    if (!kv_scale || (p->rope_dim > 0 && !k_rope_cache)) return MLA_ERR_INVALID_ARG;
  } else if (k_rope_cache || kv_scale) {
    return MLA_ERR_INVALID_ARG;
  }
  const mla::WorkspaceLayout L = layout_for(p, W);
  if (workspace_bytes < L.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (!workspace) return MLA_ERR_INVALID_ARG;
  const void* ptrs[] = {q_lat, q_rope, kv_cache, k_rope_cache, kv_scale, block_table, seq_lens, out, lse};
  const size_t need = kernel == MLA_KERNEL_SIMT ? 4 : 16;
  for (const void* q : ptrs)
    if (q && !aligned(q, need)) return MLA_ERR_ALIGNMENT;
  if (!aligned(workspace, 256)) return MLA_ERR_ALIGNMENT;

  const int dev = current_device();
  int* status = status_word(dev);
  if (!status) return MLA_ERR_CUDA;
  mla::DecodeArgs a = make_args(p, W);
  a.q_lat = q_lat;
  a.q_rope = q_rope;
  a.cache = kv_cache;
  a.k_rope = (const uint16_t*)k_rope_cache;
  a.kv_scale = kv_scale;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.out = out;
  a.lse = lse;
  char* ws = (char*)workspace;
  a.meta = (int32_t*)(ws + L.meta_off);
  a.lse_part = (float*)(ws + L.lse_off);
  a.o_part = (float*)(ws + L.o_off);
  a.status = status;
  cudaStream_t s = (cudaStream_t)stream;
  auto record = [&](int i) {
    return !events || cudaEventRecord((cudaEvent_t)events[i], s) == cudaSuccess;
  };
  if (!record(0)) return MLA_ERR_CUDA;
  cudaError_t e = kernel == MLA_KERNEL_TCGEN05   ? mla::launch_tc_decode(a, s)
                  : kernel == MLA_KERNEL_TC_PAIR ? mla::launch_pair_decode(a, s)
                                                 : mla::launch_simt_decode(a, s);
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  if (!record(1)) return MLA_ERR_CUDA;
  e = mla::launch_combine(a, s);
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  return record(2) ? MLA_OK : MLA_ERR_CUDA;
}
}  // namespace

mla_status_t mla_decode(const mla_decode_params_t* p, const void* q_lat, const void* q_rope,
                        const void* kv_cache, const void* k_rope_cache, const float* kv_scale,
                        const int32_t* block_table, const int32_t* seq_lens, void* out, float* lse,
                        void* workspace, size_t workspace_bytes, void* stream) {
  return decode_impl(p, q_lat, q_rope, kv_cache, k_rope_cache, kv_scale, block_table, seq_lens, out, lse,
                     workspace, workspace_bytes, stream, nullptr);
}

mla_status_t mla_decode_timed(const mla_decode_params_t* p, const void* q_lat, const void* q_rope,
                              const void* kv_cache, const void* k_rope_cache, const float* kv_scale,
                              const int32_t* block_table, const int32_t* seq_lens, void* out, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream, void* const* events) {
  if (!events || !events[0] || !events[1] || !events[2]) return MLA_ERR_INVALID_ARG;
  return decode_impl(p, q_lat, q_rope, kv_cache, k_rope_cache, kv_scale, block_table, seq_lens, out, lse,
                     workspace, workspace_bytes, stream, events);
}

// ---------------------------------------------------------------------------- host I/O
namespace {
struct HostIoLayout {
  size_t ws_off, ws_bytes, q_off, qr_off, bt_off, sl_off, out_off, lse_off, total;
  size_t q_bytes, qr_bytes, bt_bytes, sl_bytes, out_bytes, lse_bytes;
};

mla_status_t host_io_layout(const mla_decode_params_t* p, HostIoLayout* H) {
  size_t ws = 0;
  mla_status_t st = mla_decode_workspace_size(p, &ws);
  if (st) return st;
  const size_t rows = (size_t)p->batch * p->q_len * p->num_heads;
  H->q_bytes = rows * p->kv_rank * elem_size(p->q_dtype);
  H->qr_bytes = rows * p->rope_dim * elem_size(p->q_dtype);
  H->bt_bytes = (size_t)p->batch * p->max_blocks_per_seq * 4;
  H->sl_bytes = (size_t)p->batch * 4;
  H->out_bytes = rows * p->kv_rank * elem_size(p->out_dtype);
  H->lse_bytes = rows * 4;
  size_t o = 0;
  H->ws_off = o; H->ws_bytes = ws; o = mla::align_up(o + ws, 256);
  H->q_off = o; o = mla::align_up(o + H->q_bytes, 256);
  H->qr_off = o; o = mla::align_up(o + H->qr_bytes, 256);
  H->bt_off = o; o = mla::align_up(o + H->bt_bytes, 256);
  H->sl_off = o; o = mla::align_up(o + H->sl_bytes, 256);
  H->out_off = o; o = mla::align_up(o + H->out_bytes, 256);
  H->lse_off = o; o = mla::align_up(o + H->lse_bytes, 256);
  H->total = o;
  return MLA_OK;
}
}  // namespace

namespace {
// Sequence chunks of a host-I/O step. With several chunks, the copies of one chunk overlap the
// decode of another: host->device copies on one internal stream, the decodes on the caller's
// stream, device->host copies on a second internal stream. One chunk for small steps, where
// the extra launches would cost more than the copies they hide.
constexpr int kHostIoChunks = 4;
constexpr size_t kHostIoChunkMinBytes = size_t(8) << 20;
constexpr int kHostIoChunkMinBatch = 16;

int host_io_chunk_count(const mla_decode_params_t* p, const HostIoLayout& H) {
  const size_t io = H.q_bytes + H.qr_bytes + H.out_bytes + H.lse_bytes;
  return (p->batch >= kHostIoChunkMinBatch && io >= kHostIoChunkMinBytes) ? kHostIoChunks : 1;
}

// Per host thread and device, so the copy streams of one thread's calls stay in call order.
struct CopyStreams {
  cudaStream_t h2d = nullptr, d2h = nullptr;
};
CopyStreams* copy_streams(int dev) {
  thread_local CopyStreams S[64];
  if (dev < 0 || dev >= 64) return nullptr;
  CopyStreams& c = S[dev];
  if (!c.h2d && cudaStreamCreateWithFlags(&c.h2d, cudaStreamNonBlocking) != cudaSuccess) c.h2d = nullptr;
  if (!c.d2h && cudaStreamCreateWithFlags(&c.d2h, cudaStreamNonBlocking) != cudaSuccess) c.d2h = nullptr;
  return (c.h2d && c.d2h) ? &c : nullptr;
}

struct HostIoArgs {
  const void *q_lat, *q_rope, *kv_cache, *k_rope_cache;
  const float* kv_scale;
  const int32_t *block_table, *seq_lens;
  void* out;
  float* lse;
};

// The chunked step. Sets *ran to false, with nothing enqueued, when a chunk's staging pointers
// would break the decode's 16-byte alignment (the caller then runs the step as one chunk).
mla_status_t host_io_chunked(const mla_decode_params_t* p, const HostIoLayout& H, int K, const HostIoArgs& h,
                             char* ws, cudaStream_t s, bool* ran) {
  *ran = false;
  const int B = p->batch;
  const int nb = ((B + K - 1) / K + 3) / 4 * 4;   // sequences per chunk, a multiple of 4
  const size_t q1 = H.q_bytes / B, qr1 = H.qr_bytes / B, bt1 = H.bt_bytes / B, out1 = H.out_bytes / B,
               lse1 = H.lse_bytes / B;
  for (int b0 = 0; b0 < B; b0 += nb) {
    const size_t offs[] = {H.q_off + b0 * q1,     H.qr_off + b0 * qr1,   H.bt_off + b0 * bt1,
                           H.sl_off + b0 * size_t(4), H.out_off + b0 * out1, H.lse_off + b0 * lse1};
    for (size_t o : offs)
      if (o % 16) return MLA_OK;
  }
  CopyStreams* cs = copy_streams(current_device());
  if (!cs) return MLA_ERR_CUDA;
  cudaEvent_t ev[2 * kHostIoChunks + 2] = {};
  int nev = 0;
  auto event = [&]() -> cudaEvent_t {
    cudaEvent_t e = nullptr;
    if (cudaEventCreateWithFlags(&e, cudaEventDisableTiming) != cudaSuccess) return nullptr;
    ev[nev++] = e;
    return e;
  };
  mla_status_t st = MLA_OK;
  *ran = true;
  do {
    cudaEvent_t start = event();
    if (!start || cudaEventRecord(start, s) != cudaSuccess || cudaStreamWaitEvent(cs->h2d, start, 0) != cudaSuccess ||
        cudaStreamWaitEvent(cs->d2h, start, 0) != cudaSuccess) {
      st = MLA_ERR_CUDA;
      break;
    }
    for (int b0 = 0; b0 < B && st == MLA_OK; b0 += nb) {
      const int n = B - b0 < nb ? B - b0 : nb;
      struct Copy { void* dst; const void* src; size_t n; };
      const Copy h2d[] = {{ws + H.q_off + b0 * q1, (const char*)h.q_lat + b0 * q1, n * q1},
                          {ws + H.qr_off + b0 * qr1, (const char*)h.q_rope + b0 * qr1, n * qr1},
                          {ws + H.bt_off + b0 * bt1, (const char*)h.block_table + b0 * bt1, n * bt1},
                          {ws + H.sl_off + b0 * size_t(4), (const char*)h.seq_lens + b0 * size_t(4), n * size_t(4)}};
      for (const Copy& c : h2d)
        if (c.n && cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, cs->h2d) != cudaSuccess) st = MLA_ERR_CUDA;
      cudaEvent_t in = event(), done = event();
      if (st || !in || !done || cudaEventRecord(in, cs->h2d) != cudaSuccess || cudaStreamWaitEvent(s, in, 0) != cudaSuccess) {
        st = MLA_ERR_CUDA;
        break;
      }
      mla_decode_params_t pc = *p;
      pc.batch = n;
      st = mla_decode(&pc, ws + H.q_off + b0 * q1, p->rope_dim ? ws + H.qr_off + b0 * qr1 : nullptr, h.kv_cache,
                      h.k_rope_cache, h.kv_scale, (const int32_t*)(ws + H.bt_off + b0 * bt1),
                      (const int32_t*)(ws + H.sl_off + b0 * size_t(4)), ws + H.out_off + b0 * out1,
                      (float*)(ws + H.lse_off + b0 * lse1), ws + H.ws_off, H.ws_bytes, s);
      if (st) break;
      if (cudaEventRecord(done, s) != cudaSuccess || cudaStreamWaitEvent(cs->d2h, done, 0) != cudaSuccess ||
          cudaMemcpyAsync((char*)h.out + b0 * out1, ws + H.out_off + b0 * out1, n * out1, cudaMemcpyDeviceToHost,
                          cs->d2h) != cudaSuccess ||
          cudaMemcpyAsync((char*)h.lse + b0 * lse1, ws + H.lse_off + b0 * lse1, n * lse1, cudaMemcpyDeviceToHost,
                          cs->d2h) != cudaSuccess)
        st = MLA_ERR_CUDA;
    }
    if (st) break;
    // the caller's stream covers the whole step, the last copy back included
    cudaEvent_t end = event();
    if (!end || cudaEventRecord(end, cs->d2h) != cudaSuccess || cudaStreamWaitEvent(s, end, 0) != cudaSuccess)
      st = MLA_ERR_CUDA;
  } while (false);
  for (int i = 0; i < nev; ++i) cudaEventDestroy(ev[i]);   // released once the work that uses them is done
  return st;
}
}  // namespace

mla_status_t mla_decode_host_io_workspace_size(const mla_decode_params_t* p, size_t* bytes) {
  if (!bytes) return MLA_ERR_INVALID_ARG;
  HostIoLayout H;
  mla_status_t st = host_io_layout(p, &H);
  if (st) return st;
  *bytes = H.total;
  return MLA_OK;
}

mla_status_t mla_decode_host_io(const mla_decode_params_t* p, const void* q_lat_host, const void* q_rope_host,
                                const void* kv_cache, const void* k_rope_cache, const float* kv_scale,
                                const int32_t* block_table_host, const int32_t* seq_lens_host, void* out_host,
                                float* lse_host, void* workspace, size_t workspace_bytes, void* stream) {
  HostIoLayout H;
  mla_status_t st = host_io_layout(p, &H);
  if (st) return st;
  if (p->batch == 0) return MLA_OK;
  if (!q_lat_host || !block_table_host || !seq_lens_host || !out_host || !lse_host) return MLA_ERR_INVALID_ARG;
  if (p->rope_dim > 0 && !q_rope_host) return MLA_ERR_INVALID_ARG;
  if (!workspace) return MLA_ERR_INVALID_ARG;
  if (workspace_bytes < H.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (!aligned(workspace, 256)) return MLA_ERR_ALIGNMENT;
  char* ws = (char*)workspace;
  cudaStream_t s = (cudaStream_t)stream;
  const int K = host_io_chunk_count(p, H);
  if (K > 1) {
    const HostIoArgs h{q_lat_host, q_rope_host, kv_cache, k_rope_cache, kv_scale, block_table_host, seq_lens_host,
                       out_host, lse_host};
    bool ran = false;
    st = host_io_chunked(p, H, K, h, ws, s, &ran);
    if (ran || st) return st;
  }
  struct Copy { void* dst; const void* src; size_t n; };
  const Copy h2d[] = {{ws + H.q_off, q_lat_host, H.q_bytes},
                      {ws + H.qr_off, q_rope_host, H.qr_bytes},
                      {ws + H.bt_off, block_table_host, H.bt_bytes},
                      {ws + H.sl_off, seq_lens_host, H.sl_bytes}};
  for (const Copy& c : h2d)
    if (c.n && cudaMemcpyAsync(c.dst, c.src, c.n, cudaMemcpyHostToDevice, s) != cudaSuccess) return MLA_ERR_CUDA;
  st = mla_decode(p, ws + H.q_off, p->rope_dim ? ws + H.qr_off : nullptr, kv_cache, k_rope_cache, kv_scale,
                  (const int32_t*)(ws + H.bt_off), (const int32_t*)(ws + H.sl_off), ws + H.out_off,
                  (float*)(ws + H.lse_off), ws + H.ws_off, H.ws_bytes, stream);
  if (st) return st;
  if (cudaMemcpyAsync(out_host, ws + H.out_off, H.out_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MLA_ERR_CUDA;
  if (cudaMemcpyAsync(lse_host, ws + H.lse_off, H.lse_bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MLA_ERR_CUDA;
  return MLA_OK;
}

// ---------------------------------------------------------------------------- plan
mla_status_t mla_plan_host(const mla_decode_params_t* p, const int32_t* seq_lens_host, int32_t* seq_block_begin,
                           int32_t* seq_first_worker, int32_t* seq_num_splits) {
  int kernel = 0, W = 0;
  mla_status_t st = resolve(p, &kernel, &W);
  if (st) return st;
  if (p->batch > 0 && (!seq_lens_host || !seq_block_begin || !seq_first_worker || !seq_num_splits))
    return MLA_ERR_INVALID_ARG;
  const int64_t cap = (int64_t)p->max_blocks_per_seq * p->block_size;
  int64_t T = 0;
  for (int b = 0; b < p->batch; ++b) {
    int64_t L = seq_lens_host[b];
    if (L < 0 || L > cap) return MLA_ERR_INVALID_ARG;
    seq_block_begin[b] = (int32_t)T;
    T += (L + p->block_size - 1) / p->block_size;
  }
  if (p->batch >= 0 && seq_block_begin) seq_block_begin[p->batch] = (int32_t)T;
  const int64_t Wa = (T > 0 && T < W) ? T : W;   // active workers: each owns >= 1 block
  for (int b = 0; b < p->batch; ++b) {
    const int64_t P = seq_block_begin[b], n = seq_block_begin[b + 1] - P;
    if (n == 0) {
      seq_first_worker[b] = 0;
      seq_num_splits[b] = 0;
      continue;
    }
    // worker containing flat block x: largest w with floor(w T / Wa) <= x
    auto owner = [&](int64_t x) { return (int32_t)(((x + 1) * Wa - 1) / T); };
    seq_first_worker[b] = owner(P);
    seq_num_splits[b] = owner(P + n - 1) - owner(P) + 1;
  }
  return MLA_OK;
}

mla_status_t mla_plan_probe(const mla_decode_params_t* p, const int32_t* block_table, const int32_t* seq_lens,
                            int32_t* token_slot, int32_t* token_worker, int32_t* seq_meta, void* stream) {
  int kernel = 0, W = 0;
  mla_status_t st = resolve(p, &kernel, &W);
  if (st) return st;
  if (p->batch == 0) return MLA_OK;
  if (!block_table || !seq_lens || !token_slot || !token_worker || !seq_meta) return MLA_ERR_INVALID_ARG;
  int* status = status_word(current_device());
  if (!status) return MLA_ERR_CUDA;
  mla::DecodeArgs a = make_args(p, W);
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.meta = seq_meta;
  a.status = status;
  return mla::launch_plan_probe(a, token_slot, token_worker, (cudaStream_t)stream) == cudaSuccess ? MLA_OK
                                                                                                 : MLA_ERR_CUDA;
}

mla_status_t mla_cache_append(const mla_append_params_t* p, const void* c_new, const void* k_rope_new,
                              void* kv_cache, void* k_rope_cache, float* kv_scale, const int32_t* block_table,
                              const int32_t* seq_lens, void* stream) {
  if (!p) return MLA_ERR_INVALID_ARG;
  if (p->batch < 0 || p->q_len < 1 || p->kv_rank < 1 || p->rope_dim < 0 || p->block_size < 1 ||
      p->num_blocks < 0 || p->max_blocks_per_seq < 1 || p->reserved != 0 || (p->rope != 0 && p->rope != 1))
    return MLA_ERR_INVALID_ARG;
  if (p->batch > 0 && p->num_blocks < 1) return MLA_ERR_INVALID_ARG;
  const bool pair_ok = (p->in_dtype == MLA_DTYPE_F32 && p->cache_dtype == MLA_DTYPE_F32) ||
                       (p->in_dtype == MLA_DTYPE_BF16 &&
                        (p->cache_dtype == MLA_DTYPE_BF16 || p->cache_dtype == MLA_DTYPE_E4M3));
  if (!pair_ok) return MLA_ERR_INVALID_ARG;
  if (p->cache_dtype == MLA_DTYPE_E4M3 && (p->kv_rank % 2 != 0 || !k_rope_cache || !kv_scale))
    return MLA_ERR_INVALID_ARG;
  if (p->rope && (p->rope_dim % 2 != 0 || !std::isfinite(p->rope_base) || !(p->rope_base > 0.f)))
    return MLA_ERR_INVALID_ARG;
  if (p->batch == 0) return MLA_OK;
  if (!c_new || !kv_cache || !block_table || !seq_lens || (p->rope_dim > 0 && !k_rope_new))
    return MLA_ERR_INVALID_ARG;
  if ((int64_t)p->max_blocks_per_seq * p->block_size > (1ll << 30)) return MLA_ERR_UNSUPPORTED;
  int* status = status_word(current_device());
  if (!status) return MLA_ERR_CUDA;
  mla::AppendArgs a{};
  a.B = p->batch;
  a.Sq = p->q_len;
  a.r = p->kv_rank;
  a.d_r = p->rope_dim;
  a.bs = p->block_size;
  a.num_blocks = p->num_blocks;
  a.max_blocks = p->max_blocks_per_seq;
  a.in_dtype = p->in_dtype;
  a.cache_dtype = p->cache_dtype;
  a.rope = p->rope;
  a.rope_base = p->rope_base;
  a.c_new = c_new;
  a.k_new = k_rope_new;
  a.cache = kv_cache;
  a.k_rope = (uint16_t*)k_rope_cache;
  a.kv_scale = kv_scale;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.status = status;
  return mla::launch_cache_append(a, (cudaStream_t)stream) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status_t mla_head_gemm(const mla_head_gemm_params_t* p, const void* x, const void* w, void* y, void* stream) {
  if (!p || p->rows < 0 || p->heads < 1 || p->k < 64 || p->n < 64 || p->k % 64 != 0 || p->n % 64 != 0 ||
      p->reserved != 0)
    return MLA_ERR_INVALID_ARG;
  if (p->heads > 65535 || (p->rows + 127) / 128 > 65535) return MLA_ERR_UNSUPPORTED;
  if (p->rows == 0) return MLA_OK;
  if (!x || !w || !y) return MLA_ERR_INVALID_ARG;
  if (((uintptr_t)x | (uintptr_t)w | (uintptr_t)y) & 15) return MLA_ERR_ALIGNMENT;
  int* status = status_word(current_device());
  if (!status) return MLA_ERR_CUDA;
  mla::GemmArgs a{};
  a.rows = p->rows;
  a.heads = p->heads;
  a.k = p->k;
  a.n = p->n;
  a.x = x;
  a.w = w;
  a.y = y;
  a.status = status;
  return mla::launch_head_gemm(a, (cudaStream_t)stream) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

// ---------------------------------------------------------------------------- sparse attention
namespace {
mla_status_t check_dsa(const mla_dsa_params_t* p) {
  if (!p) return MLA_ERR_INVALID_ARG;
  if (p->batch < 0 || p->q_len < 1 || p->index_heads < 1 || p->index_dim < 1 || p->block_size < 1 ||
      p->num_blocks < 0 || p->max_blocks_per_seq < 1 || p->max_seq_len < 0 || p->top_k < 1 ||
      (p->causal != 0 && p->causal != 1) || p->reserved != 0)
    return MLA_ERR_INVALID_ARG;
  if (p->batch > 0 && p->num_blocks < 1) return MLA_ERR_INVALID_ARG;
  if (p->index_heads != mla::kDsaHeads || p->index_dim != mla::kDsaDim || p->block_size != 64)
    return MLA_ERR_UNSUPPORTED;
  if ((int64_t)p->batch * p->q_len > 65535) return MLA_ERR_UNSUPPORTED;   // one grid row per query row
  if ((int64_t)p->max_blocks_per_seq * p->block_size > (1ll << 30)) return MLA_ERR_UNSUPPORTED;
  if ((int64_t)p->num_blocks * p->block_size > (1ll << 31) - 1) return MLA_ERR_UNSUPPORTED;
  return MLA_OK;
}

mla::DsaArgs dsa_args(const mla_dsa_params_t* p, int* status) {
  mla::DsaArgs a{};
  a.B = p->batch;
  a.Sq = p->q_len;
  a.bs = p->block_size;
  a.num_blocks = p->num_blocks;
  a.max_blocks = p->max_blocks_per_seq;
  a.max_seq_len = p->max_seq_len;
  a.top_k = p->top_k;
  a.causal = p->causal;
  a.status = status;
  return a;
}
}  // namespace

mla_status_t mla_dsa_index(const mla_dsa_params_t* p, const void* q_codes, const float* q_scale,
                           const float* weights, const void* k_codes, const float* k_scale,
                           const int32_t* block_table, const int32_t* seq_lens, float* scores, void* stream) {
  mla_status_t st = check_dsa(p);
  if (st) return st;
  if (p->batch == 0 || p->max_seq_len == 0) return MLA_OK;
  if (!q_codes || !q_scale || !weights || !k_codes || !k_scale || !block_table || !seq_lens || !scores)
    return MLA_ERR_INVALID_ARG;
  if (!aligned(q_codes, 16) || !aligned(k_codes, 16) || !aligned(k_scale, 16)) return MLA_ERR_ALIGNMENT;
  const void* p4[] = {q_scale, weights, block_table, seq_lens, scores};
  for (const void* q : p4)
    if (!aligned(q, 4)) return MLA_ERR_ALIGNMENT;
  int* status = status_word(current_device());
  if (!status) return MLA_ERR_CUDA;
  mla::DsaArgs a = dsa_args(p, status);
  a.q = (const uint8_t*)q_codes;
  a.q_scale = q_scale;
  a.w = weights;
  a.k = (const uint8_t*)k_codes;
  a.k_scale = k_scale;
  a.block_table = block_table;
  a.seq_lens = seq_lens;
  a.scores = scores;
  return mla::launch_dsa_index(a, (cudaStream_t)stream) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status_t mla_dsa_topk(const mla_dsa_params_t* p, const float* scores, const int32_t* seq_lens,
                          int32_t* indices, int32_t* counts, void* stream) {
  mla_status_t st = check_dsa(p);
  if (st) return st;
  if (p->batch == 0) return MLA_OK;
  if (!scores || !seq_lens || !indices || !counts) return MLA_ERR_INVALID_ARG;
  const void* p4[] = {scores, seq_lens, indices, counts};
  for (const void* q : p4)
    if (!aligned(q, 4)) return MLA_ERR_ALIGNMENT;
  int* status = status_word(current_device());
  if (!status) return MLA_ERR_CUDA;
  mla::DsaArgs a = dsa_args(p, status);
  a.scores = (float*)scores;
  a.seq_lens = seq_lens;
  a.indices = indices;
  a.counts = counts;
  return mla::launch_dsa_topk(a, (cudaStream_t)stream) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status_t mla_sparse_decode(const mla_decode_params_t* p, int32_t top_k, const void* q_lat,
                               const void* q_rope, const void* kv_cache, const int32_t* block_table,
                               const int32_t* indices, const int32_t* counts, void* out, float* lse,
                               void* workspace, size_t workspace_bytes, void* stream) {
  int kernel = 0, W = 0;
  mla_status_t st = resolve(p, &kernel, &W, true);
  if (st) return st;
  if (top_k < 1) return MLA_ERR_INVALID_ARG;
  if (p->q_len != 1 || p->causal != 0 || p->cache_dtype != MLA_DTYPE_BF16 ||
      (kernel != MLA_KERNEL_TCGEN05 && kernel != MLA_KERNEL_TC_PAIR))
    return MLA_ERR_UNSUPPORTED;
  if (p->batch == 0) return MLA_OK;
  if (!q_lat || !q_rope || !kv_cache || !block_table || !indices || !counts || !out || !lse)
    return MLA_ERR_INVALID_ARG;
  const mla::WorkspaceLayout L = layout_for(p, W);
  if (workspace_bytes < L.total) return MLA_ERR_WORKSPACE_TOO_SMALL;
  if (!workspace) return MLA_ERR_INVALID_ARG;
  const void* ptrs[] = {q_lat, q_rope, kv_cache, block_table, out, lse};
  for (const void* q : ptrs)
    if (!aligned(q, 16)) return MLA_ERR_ALIGNMENT;
  if (!aligned(indices, 4) || !aligned(counts, 4) || !aligned(workspace, 256)) return MLA_ERR_ALIGNMENT;
  int* status = status_word(current_device());
  if (!status) return MLA_ERR_CUDA;
  mla::DecodeArgs a = make_args(p, W);
  a.q_lat = q_lat;
  a.q_rope = q_rope;
  a.cache = kv_cache;
  a.block_table = block_table;
  a.seq_lens = counts;   // each sequence's length is its list's count
  a.sel_idx = indices;
  a.top_k = top_k;
  if (top_k < a.len_cap) a.len_cap = top_k;   // a count above top_k is an error (and is clamped)
  a.out = out;
  a.lse = lse;
  char* ws = (char*)workspace;
  a.meta = (int32_t*)(ws + L.meta_off);
  a.lse_part = (float*)(ws + L.lse_off);
  a.o_part = (float*)(ws + L.o_off);
  a.status = status;
  cudaStream_t s = (cudaStream_t)stream;
  const cudaError_t e = kernel == MLA_KERNEL_TC_PAIR ? mla::launch_pair_decode(a, s) : mla::launch_tc_decode(a, s);
  if (e != cudaSuccess) return MLA_ERR_CUDA;
  return mla::launch_combine(a, s) == cudaSuccess ? MLA_OK : MLA_ERR_CUDA;
}

mla_status_t mla_get_device_status(void* stream, int32_t* device_status) {
  if (!device_status) return MLA_ERR_INVALID_ARG;
  if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return MLA_ERR_CUDA;
  int* status = status_word(current_device());
  if (!status) return MLA_ERR_CUDA;
  int v = 0;
  if (cudaMemcpy(&v, status, sizeof v, cudaMemcpyDeviceToHost) != cudaSuccess) return MLA_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpy(status, &zero, sizeof zero, cudaMemcpyHostToDevice) != cudaSuccess) return MLA_ERR_CUDA;
  *device_status = v;
  return MLA_OK;
}

}  // extern "C"
