/*
 * mla_decode.h -- C ABI of the B200 (sm_100a) absorbed multi-head latent attention
 * (MLA) decode library, libmla_decode.so.
 *
 * The operation. One decode step of one attention layer for a batch of sequences
 * whose keys and values live in a shared compressed latent cache:
 *
 *   for every sequence b, query position s < Sq, head h:
 *     sigma_t = softmax_scale * ( q_lat[b,s,h,:] . c_t  +  q_rope[b,s,h,:] . kR_t )
 *     lse[b,s,h]   = log sum_t exp(sigma_t)                      (natural log)
 *     out[b,s,h,:] = sum_t exp(sigma_t - lse[b,s,h]) * c_t
 *
 *   c_t (kv_rank = r values) is token t's cached latent and serves as both the key
 *   content and the value; kR_t (rope_dim = d_r values) is its decoupled RoPE key,
 *   shared by all heads. q_lat is the absorbed query (W^UK folded into the query
 *   projection) and q_rope the RoPE part of the query.
 *   Sources: "TransMLA: Multi-Head Latent Attention Is All You Need" (paper-graph
 *   summary), sec. 3.4.5 "The full MLA structure after conversion" (absorbed query
 *   [(W^UK_i)^T q; q^R] against the cached [c^KV; k^R]); TPLA paper-graph summary,
 *   sec. 3.4, eq. 5 (softmax(Q c^T) c: the latent is the value) and "The RoPE
 *   handling" (score = (Q c^T + q^PE k^PE^T) / sqrt(d_h + d_r)). The caller passes the
 *   scale, so any of the pages' temperature conventions can be used.
 *
 *   Attended tokens: with causal == 0 every query row sees tokens [0, seq_lens[b]).
 *   With causal != 0 the Sq queries are the last Sq tokens of the sequence and query
 *   s sees tokens [0, seq_lens[b] - Sq + 1 + s). A row that sees no token gets
 *   out = 0 and lse = -inf.
 *
 * Cache layout (paged). Token t of sequence b is slot t % block_size of physical
 * block block_table[b * max_blocks_per_seq + t / block_size].
 *   cache_dtype F32 / BF16: kv_cache = [num_blocks, block_size, r + d_r], latent then
 *     RoPE key, row-major. k_rope_cache and kv_scale must be NULL.
 *   cache_dtype E4M3 (OCP FP8 e4m3, no infinities): kv_cache = codes
 *     [num_blocks, block_size, r] (uint8); c_t = decode(code) * kv_scale[slot];
 *     k_rope_cache = bf16 [num_blocks, block_size, d_r]; kv_scale = f32
 *     [num_blocks, block_size].
 *   Slots past a sequence's length in its last block are never read for scores or
 *   values (they may hold anything, NaN included).
 *
 * Other tensors (all contiguous, row-major, device-resident unless stated):
 *   q_lat  [B, Sq, H, r]   q_dtype        q_rope [B, Sq, H, d_r] q_dtype
 *   block_table [B, max_blocks_per_seq] int32     seq_lens [B] int32
 *   out    [B, Sq, H, r]   out_dtype      lse    [B, Sq, H] float32
 * Supported dtype triples (q, cache, out): (F32, F32, F32), (BF16, BF16, BF16|F32),
 * (BF16, E4M3, BF16|F32).
 *
 * Ownership and threading. The caller owns every buffer, the workspace included;
 * the library never allocates device memory. Calls are stream-ordered and
 * asynchronous: they enqueue work on `stream` (a cudaStream_t, NULL = legacy default
 * stream) on the current device and return. Concurrent calls on different streams
 * need different workspaces.
 *
 * Errors. Argument errors are detected on the host before anything is enqueued and
 * returned synchronously (nothing is launched). A failed launch returns MLA_ERR_CUDA.
 * Data-dependent errors found on the device do not stop the other sequences of the
 * call, and they are visible in the output: every row (out and lse) of a sequence whose
 * seq_len is outside [0, max_blocks_per_seq * block_size], or whose block table names a
 * block outside [0, num_blocks) within its length, is written as NaN; so is every row a
 * kernel did not finish because one of its bounded waits ran out (see
 * mla_set_wait_timeout_ns). A sticky per-device status word records the first such
 * error (MLA_ERR_BAD_SEQ_LEN, MLA_ERR_BAD_BLOCK_ID, MLA_ERR_TIMEOUT);
 * mla_get_device_status() reads and clears it. No device code traps, and the context
 * stays usable.
 */
#ifndef MLA_DECODE_H_
#define MLA_DECODE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define MLA_DECODE_ABI_VERSION 1

typedef enum { MLA_DTYPE_F32 = 0, MLA_DTYPE_BF16 = 1, MLA_DTYPE_E4M3 = 2 } mla_dtype_t;

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARG = 1,         /* bad shape, NULL pointer, bad dtype combination */
  MLA_ERR_UNSUPPORTED = 2,         /* valid request that the chosen kernel cannot run */
  MLA_ERR_ALIGNMENT = 3,           /* a device pointer is not 16-byte aligned */
  MLA_ERR_WORKSPACE_TOO_SMALL = 4,
  MLA_ERR_CUDA = 5,                /* CUDA runtime / launch error */
  MLA_ERR_BAD_BLOCK_ID = 6,        /* device-detected, sticky */
  MLA_ERR_BAD_SEQ_LEN = 7,         /* device-detected, sticky */
  MLA_ERR_TIMEOUT = 8              /* device-detected bounded wait expiry, sticky */
} mla_status_t;

typedef enum {
  MLA_KERNEL_AUTO = 0,     /* tensor-core kernel when the shape allows it (TC_PAIR for a bf16 cache,
                              TCGEN05 for an FP8 cache and for sparse decode), else SIMT */
  MLA_KERNEL_SIMT = 1,     /* fp32 CUDA-core kernel: any r <= 1024, r + d_r <= 1280 */
  MLA_KERNEL_TCGEN05 = 2,  /* tcgen05/TMA kernel: r = 512, d_r = 64, block_size = 64 */
  MLA_KERNEL_TC_PAIR = 3   /* split-role tcgen05/TMA kernel on CTA pairs (scores on one CTA, P.V on its
                              peer): the shapes of MLA_KERNEL_TCGEN05 with a bf16 cache */
} mla_kernel_t;

typedef struct {
  int32_t batch;               /* B >= 0 */
  int32_t q_len;               /* Sq >= 1 query tokens per sequence */
  int32_t num_heads;           /* H >= 1 */
  int32_t kv_rank;             /* r >= 1, latent width */
  int32_t rope_dim;            /* d_r >= 0, decoupled RoPE key width */
  int32_t block_size;          /* tokens per cache block */
  int32_t num_blocks;          /* physical blocks in the cache */
  int32_t max_blocks_per_seq;  /* row stride of block_table */
  int32_t q_dtype;             /* mla_dtype_t */
  int32_t cache_dtype;         /* mla_dtype_t */
  int32_t out_dtype;           /* mla_dtype_t */
  int32_t causal;              /* 0 / 1, see above */
  float softmax_scale;         /* multiplies the summed score; finite */
  int32_t num_workers;         /* 0 = auto; else the number of KV-range workers */
  int32_t kernel;              /* mla_kernel_t */
  int32_t reserved;            /* must be 0 */
} mla_decode_params_t;

/* Bytes of device workspace mla_decode needs for these parameters (host only; with
 * num_workers == 0 it queries the current device's SM count). The bound does not
 * depend on seq_lens. */
mla_status_t mla_decode_workspace_size(const mla_decode_params_t* params, size_t* bytes);

/* Kernel and worker count a call with these parameters would use (host only). */
mla_status_t mla_decode_resolve(const mla_decode_params_t* params, int32_t* kernel,
                                int32_t* num_workers);

/* Enqueue one decode step (see the header comment). All tensor pointers are device
 * pointers. workspace must hold mla_decode_workspace_size() bytes, 256-byte aligned;
 * its contents need no initialisation and are clobbered. */
mla_status_t mla_decode(const mla_decode_params_t* params, const void* q_lat, const void* q_rope,
                        const void* kv_cache, const void* k_rope_cache, const float* kv_scale,
                        const int32_t* block_table, const int32_t* seq_lens, void* out, float* lse,
                        void* workspace, size_t workspace_bytes, void* stream);

/* mla_decode, plus three CUDA events (cudaEvent_t, created by the caller) recorded on
 * `stream`: events[0] before the decode kernel, events[1] between the decode kernel
 * and the split-combine kernel, events[2] after the combine. Lets a caller time each
 * kernel of the step on the launching stream; the work done is identical. */
mla_status_t mla_decode_timed(const mla_decode_params_t* params, const void* q_lat, const void* q_rope,
                              const void* kv_cache, const void* k_rope_cache, const float* kv_scale,
                              const int32_t* block_table, const int32_t* seq_lens, void* out, float* lse,
                              void* workspace, size_t workspace_bytes, void* stream,
                              void* const* events);

/* Bytes of device workspace mla_decode_host_io needs: device staging for the per-step
 * inputs and outputs plus mla_decode's own workspace. */
mla_status_t mla_decode_host_io_workspace_size(const mla_decode_params_t* params, size_t* bytes);

/* One decode step whose per-step tensors are in HOST memory (pinned memory makes the
 * copies asynchronous): q_lat, q_rope, block_table, seq_lens are copied to the
 * device, the step runs, out and lse are copied back. The cache (kv_cache,
 * k_rope_cache, kv_scale) stays device-resident. The call returns once the work is
 * enqueued; synchronise `stream` before reading out / lse (the stream's work covers the
 * whole step, the copies back included).
 * A step of at least 16 sequences whose per-step copies (q_lat, q_rope, out, lse) reach
 * 8 MiB runs as four chunks of consecutive sequences (a multiple of 4 each): the copies
 * of one chunk overlap the decode of another, on two copy streams the library keeps per
 * host thread and device, ordered against `stream` by events. Each chunk is a decode of
 * its own (its own split of the sequences over the workers), so such a step can differ
 * from one mla_decode over the whole batch in the last bits, within the decode's
 * accuracy; smaller steps run as one chunk on `stream` and match mla_decode exactly. */
mla_status_t mla_decode_host_io(const mla_decode_params_t* params, const void* q_lat_host,
                                const void* q_rope_host, const void* kv_cache,
                                const void* k_rope_cache, const float* kv_scale,
                                const int32_t* block_table_host, const int32_t* seq_lens_host,
                                void* out_host, float* lse_host, void* workspace,
                                size_t workspace_bytes, void* stream);

/* Largest workspace, in bytes, that mla_decode_noalloc can serve (64 MiB). */
#define MLA_NOALLOC_SCRATCH_BYTES (64u << 20)

/* mla_decode for callers that cannot allocate device memory on the decode path (a
 * serving engine that has reserved the GPU's memory for its cache, a plugin running in
 * a memory pool it does not own). The paper has no counterpart to this entry point: it
 * is a convenience of the library, not a step of the method. The split workspace is a file-scope device array of
 * MLA_NOALLOC_SCRATCH_BYTES that every GPU loading the library keeps until exit.
 * Arguments are those of mla_decode without the workspace. The first call on each
 * device looks up that device's array address (make it before any stream capture).
 * Returns MLA_ERR_WORKSPACE_TOO_SMALL, with nothing launched, when
 * mla_decode_workspace_size() exceeds MLA_NOALLOC_SCRATCH_BYTES. Allocates nothing.
 * All calls on a device share the array: calls whose GPU work overlaps race, so
 * serialise them (one stream, or external ordering). */
mla_status_t mla_decode_noalloc(const mla_decode_params_t* params, const void* q_lat, const void* q_rope,
                                const void* kv_cache, const void* k_rope_cache, const float* kv_scale,
                                const int32_t* block_table, const int32_t* seq_lens, void* out, float* lse,
                                void* stream);

/* MLA_NOALLOC_SCRATCH_BYTES as compiled into the loaded library. */
size_t mla_decode_noalloc_max_workspace(void);

/* Split plan on the host, for tests. Work is the flat list of cache blocks of all
 * sequences in batch order; with W' = min(W, T) active workers, worker w < W' owns
 * blocks [floor(w*T/W'), floor((w+1)*T/W')) of the T blocks (at least one each). Outputs (host arrays): seq_block_begin[B + 1] (prefix of blocks per
 * sequence), seq_first_worker[B] and seq_num_splits[B] (workers that touch each
 * sequence; 0 splits for an empty sequence). W comes from mla_decode_resolve. */
mla_status_t mla_plan_host(const mla_decode_params_t* params, const int32_t* seq_lens_host,
                           int32_t* seq_block_begin, int32_t* seq_first_worker,
                           int32_t* seq_num_splits);

/* Device probe of the same plan, for tests: every worker walks its block range with
 * the device code the decode kernels use and records, for each logical token t of
 * sequence b, the physical slot it reads (block * block_size + offset) in
 * token_slot[b * max_blocks_per_seq * block_size + t] and its worker id in
 * token_worker[...]; unread entries are left untouched. seq_meta[2 * b] and
 * seq_meta[2 * b + 1] receive the first worker and split count the kernels use.
 * All pointers are device pointers. */
mla_status_t mla_plan_probe(const mla_decode_params_t* params, const int32_t* block_table,
                            const int32_t* seq_lens, int32_t* token_slot, int32_t* token_worker,
                            int32_t* seq_meta, void* stream);

/* Synchronise `stream`, then read and clear the current device's sticky status word
 * (MLA_OK or one of the device-detected codes). Returns MLA_ERR_CUDA if the
 * synchronisation itself failed. */
mla_status_t mla_get_device_status(void* stream, int32_t* device_status);

/* Limit, in nanoseconds, of every bounded wait inside the library's kernels (pipeline
 * hand-offs between warps and between the CTAs of a cluster). Default 2e9 (2 s); 0
 * restores the default. A wait that runs out ends its kernel's work early: the rows it
 * did not finish are NaN and MLA_ERR_TIMEOUT is recorded in the status word. The waits
 * that let already-issued copies and MMAs complete before a CTA exits keep a limit of at
 * least 2 s, so a short limit never leaves work in flight. Process-wide; it applies to
 * launches enqueued after the call (meant for tests and watchdogs). No counterpart in the
 * papers: it is a property of this library's kernels. */
mla_status_t mla_set_wait_timeout_ns(uint64_t ns);
/* The limit currently in force. */
uint64_t mla_get_wait_timeout_ns(void);

/* Static, human-readable name of a status code. */
const char* mla_status_string(int32_t status);

/* ------------------------------------------------------------------ cache append
 *
 * Writes the latent and RoPE key of the Sq new tokens of every sequence into the paged
 * cache that mla_decode reads ("TransMLA: Multi-Head Latent Attention Is All You Need",
 * sec. 3.4.5: the cache holds one latent c and one decoupled RoPE key kR per token, and
 * the RoPE key is recomputed for the new token at its position; the "Watching the fusion
 * actually fail, on numbers" passage of the TransMLA & Sparse Latent Attention lesson shows
 * the position rotation R(t) on a two-dimensional toy).
 *
 * Token s of sequence b has logical position pos = seq_lens[b] - Sq + s (the Sq new tokens
 * are the last Sq of seq_lens[b], the convention of mla_decode's causal mode) and goes to
 * physical block block_table[b][pos / block_size], slot pos % block_size.
 *   - in_dtype MLA_F32 -> cache_dtype MLA_F32, or MLA_BF16 -> MLA_BF16: the values are stored
 *     as given ([num_blocks][block_size][r + d_r]).
 *   - in_dtype MLA_BF16 -> cache_dtype MLA_E4M3: the latent is quantised per token:
 *     scale = max_k |c_k| / 448 (fp32 division), code_k = e4m3(c_k / scale) (fp32 division,
 *     round to nearest even, saturated to +-448; OCP FP8 e4m3, no infinities); scale 0 (an
 *     all-zero latent) stores zero codes. Codes go to kv_cache [num_blocks][block_size][r],
 *     the scale to kv_scale [num_blocks][block_size], the bf16 RoPE key to k_rope_cache
 *     [num_blocks][block_size][d_r].
 *   - rope != 0: the RoPE key is rotated before it is stored: pairs (x[2i], x[2i+1]) turn by
 *     pos * theta_i with theta_i = rope_base^(-2i / d_r) (angle and rotation in fp64, result
 *     rounded to the cache type). rope == 0 stores k_rope_new as given (already rotated).
 *
 * c_new [B, Sq, r] and k_rope_new [B, Sq, d_r] have type in_dtype; all pointers are device
 * pointers; the call is asynchronous on `stream` and allocates nothing. Argument errors
 * return at once without a launch. A token whose position is negative or past the block
 * table raises MLA_ERR_BAD_SEQ_LEN, one whose block id is out of range MLA_ERR_BAD_BLOCK_ID
 * (sticky device status word, read with mla_get_device_status); such tokens are not
 * written. Tokens of different sequences must map to different slots. */
typedef struct {
  int32_t batch;               /* B */
  int32_t q_len;               /* Sq: new tokens per sequence */
  int32_t kv_rank;             /* r */
  int32_t rope_dim;            /* d_r (even when rope != 0) */
  int32_t block_size;
  int32_t num_blocks;
  int32_t max_blocks_per_seq;  /* row stride of block_table */
  int32_t in_dtype;            /* mla_dtype_t of c_new and k_rope_new */
  int32_t cache_dtype;         /* mla_dtype_t of the cache */
  int32_t rope;                /* 0: store k_rope_new as given; 1: rotate it first */
  float rope_base;             /* theta base of the rotation, e.g. 10000 */
  int32_t reserved;            /* must be 0 */
} mla_append_params_t;

mla_status_t mla_cache_append(const mla_append_params_t* params, const void* c_new, const void* k_rope_new,
                              void* kv_cache, void* k_rope_cache, float* kv_scale, const int32_t* block_table,
                              const int32_t* seq_lens, void* stream);

/* ------------------------------------------------------------------ per-head GEMM
 *
 * y[m, h, :] = x[m, h, :] . w[h] for m < rows and every head h: bf16 operands, fp32
 * accumulation, bf16 result (round to nearest even). The two weight products around the
 * absorbed decode are instances ("TransMLA: Multi-Head Latent Attention Is All You Need",
 * sec. 3.4.5, the full MLA structure after conversion: W^UK is absorbed into the query and
 * W^UV applied to the attention output):
 *   query absorption     x = q_nope [rows, H, d_h], w[h] = W^UK_h (d_h x r)    -> y = q_lat [rows, H, r]
 *   output up-projection x = out    [rows, H, r],   w[h] = W^UV_h^T (r x d_v)  -> y [rows, H, d_v]
 * with rows = B * Sq. Layouts: x [rows][heads][k], w [heads][k][n], y [rows][heads][n],
 * contiguous device arrays, 16-byte aligned; k and n multiples of 64. Tensor cores (tcgen05,
 * M = 128 rows per tile, K = 64 per staged chunk). Asynchronous on `stream`, allocates
 * nothing. Argument errors return at once; a wait timeout sets the sticky status word. */
typedef struct {
  int32_t rows;      /* m extent (B * Sq) */
  int32_t heads;     /* H */
  int32_t k;         /* contraction length per head */
  int32_t n;         /* output width per head */
  int32_t reserved;  /* must be 0 */
} mla_head_gemm_params_t;

mla_status_t mla_head_gemm(const mla_head_gemm_params_t* params, const void* x, const void* w, void* y,
                           void* stream);

/* ------------------------------------------------------------------ sparse attention (DSA)
 *
 * DeepSeek Sparse Attention on the same paged cache ("TransMLA & Sparse Latent Attention"
 * lesson, Chapter 6 "The lightning indexer" and "Fine-grained token selection"; Chapter 7
 * "The indexer keeps its own small cache" and "DSA runs in MLA's MQA mode"). One sparse
 * decode step is three calls on one stream:
 *
 *   mla_dsa_index   scores[b,s,t] = sum_j w[b,s,j] * ReLU( q_j . k_t ) for every token t
 *                   query row (b, s) sees (the decode's causal rule), j < index_heads;
 *                   q_j = e4m3(q_codes[b,s,j,:]) * q_scale[b,s,j],
 *                   k_t = e4m3(k_codes[slot(t),:]) * k_scale[slot(t)], slot(t) through the
 *                   block table. Entries t >= that count are not written.
 *   mla_dsa_topk    for each row, the positions of its top_k highest scores (all of them
 *                   when it sees top_k or fewer tokens), ascending, -1 past the count;
 *                   equal scores at the cut go to the lower positions (-0 equals +0).
 *                   counts[b,s] = min(seen, top_k).
 *   mla_sparse_decode  the decode above over each sequence's selected positions only
 *                   (q_len 1, bf16 cache, tensor-core kernel): row (b, 0, h) attends
 *                   exactly tokens indices[b, 0 .. counts[b]).
 *
 * Tensors (device, contiguous): q_codes uint8 [B, Sq, index_heads, index_dim] and
 * k_codes uint8 [num_blocks, block_size, index_dim] (the indexer's key side-cache, paged
 * like the latent cache), both 16-byte aligned; q_scale, weights f32 [B, Sq, index_heads];
 * k_scale f32 [num_blocks, block_size], 16-byte aligned (scales >= 0: the kernel folds them
 * out of the ReLU); scores f32 [B, Sq, max_seq_len];
 * indices int32 [B, Sq, top_k]; counts int32 [B, Sq]. The tensor path has index_heads 64,
 * index_dim 128, block_size 64 (MLA_ERR_UNSUPPORTED otherwise). A seq_len above
 * max_seq_len or the block table's capacity sets MLA_ERR_BAD_SEQ_LEN on the device (that
 * row is skipped); a block id out of range sets MLA_ERR_BAD_BLOCK_ID (its tokens score
 * NaN; in the sparse decode they read as zeros). Positions handed to the sparse decode
 * must be below their sequence's length. Asynchronous, allocates nothing. */
typedef struct {
  int32_t batch;               /* B */
  int32_t q_len;               /* Sq */
  int32_t index_heads;         /* H^I (64) */
  int32_t index_dim;           /* d^I (128) */
  int32_t block_size;          /* 64 */
  int32_t num_blocks;
  int32_t max_blocks_per_seq;  /* row stride of block_table */
  int32_t max_seq_len;         /* row stride of scores; >= every seq_len */
  int32_t top_k;               /* k (2048 in DeepSeek-V3.2) */
  int32_t causal;              /* 0 or 1, as in the decode */
  int32_t reserved;            /* must be 0 */
} mla_dsa_params_t;

mla_status_t mla_dsa_index(const mla_dsa_params_t* params, const void* q_codes, const float* q_scale,
                           const float* weights, const void* k_codes, const float* k_scale,
                           const int32_t* block_table, const int32_t* seq_lens, float* scores, void* stream);

mla_status_t mla_dsa_topk(const mla_dsa_params_t* params, const float* scores, const int32_t* seq_lens,
                          int32_t* indices, int32_t* counts, void* stream);

/* The decode's params (q_len 1, causal 0, BF16 cache, kernel AUTO, TC_PAIR or TCGEN05) and
 * workspace (mla_decode_workspace_size of the same params). indices [B, top_k] int32,
 * counts [B] int32, device. The kernel reads indices[b, 0 .. counts[b]) and checks each
 * position against the block table; a count outside [0, top_k] is clamped into it and, like
 * a bad position, sets the sticky status (MLA_ERR_BAD_SEQ_LEN / MLA_ERR_BAD_BLOCK_ID) and makes
 * that sequence's rows NaN (mla_dsa_topk's outputs always satisfy it). */
mla_status_t mla_sparse_decode(const mla_decode_params_t* params, int32_t top_k, const void* q_lat,
                               const void* q_rope, const void* kv_cache, const int32_t* block_table,
                               const int32_t* indices, const int32_t* counts, void* out, float* lse,
                               void* workspace, size_t workspace_bytes, void* stream);

/* MLA_DECODE_ABI_VERSION of the loaded library. */
int32_t mla_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MLA_DECODE_H_ */
