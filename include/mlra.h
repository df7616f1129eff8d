/*
 * mlra.h - C ABI of the B200 (sm_100a) decode path for Multi-Head Low-Rank Attention.
 *
 * The operation (one decode step, one new query token per sequence):
 *   Each cached token holds one latent c = [c_1 | ... | c_k] cut into k blocks of width
 *   d_b = d_c / k, plus one decoupled RoPE key k^R of width d_rope shared by every head
 *   ("Multi-Head Low-Rank Attention: Making Compressed Attention Actually Parallelizable",
 *   Core Mechanism and Framework Shift; "Multi-Head Low-Rank Attention" abstract). Head group
 *   j = heads [j*h/k, (j+1)*h/k) attends only to block c_j. For head h in group j:
 *     q~_h  = (W^UK_h)^T q^C_h                       query absorption (lesty.tech MLA article,
 *                                                    section 5; ai360xpert "Absorbing the
 *                                                    up-projection")
 *     s_t   = scale * (q~_h . c_j[t] + q^R_h . k^R[t])   decoupled RoPE score (lesty.tech, section 4)
 *     o~_h  = sum_t softmax(s)_t c_j[t]               value accumulated in latent space
 *     o_h   = W^UV_h o~_h                             one final up-projection (lesty.tech, section 5)
 *   k = 1 is plain MLA (lesty.tech sections 3-5; Table 1 of the MLRA paper page, MLA row).
 *
 * Conventions shared by every entry point:
 *   - Device pointers are CUDA global memory on the current device; host pointers are marked.
 *   - The caller owns every buffer. The library allocates no device memory: scratch lives in
 *     the caller's workspace (mlra_workspace_size), except for mlra_decode_noalloc, whose
 *     scratch is one fixed 16 MiB device array of the library. A handle borrows the weight
 *     pointers until mlra_destroy.
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default stream). No entry
 *     point synchronises, except mlra_get_status.
 *   - Return values are mlra_status codes. Argument errors are found on the host before any
 *     launch. Errors that only the device can see (a page id outside the pool, a sequence
 *     longer than its page-table row, a pipeline wait that timed out) are written to a
 *     device status word that mlra_get_status reads after the stream has been synchronised.
 *     No kernel traps.
 *   - Calls on different streams are safe when each uses its own workspace.
 *   - All symbol names are plain ASCII.
 */
#ifndef MLRA_H_
#define MLRA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLRA_OK = 0,
  MLRA_ERR_INVALID_ARG = -1,   /* null pointer, bad size, inconsistent dims */
  MLRA_ERR_UNSUPPORTED = -2,   /* dims outside the compiled kernel set, or not an sm_100 GPU */
  MLRA_ERR_CUDA = -3,          /* a CUDA runtime call failed */
  MLRA_ERR_PAGE_OOB = -4,      /* device: a page-table entry outside [0, num_pages) */
  MLRA_ERR_TIMEOUT = -5,       /* device: a pipeline wait passed its time limit */
  MLRA_ERR_WORKSPACE = -6,     /* workspace smaller than mlra_workspace_size */
  MLRA_ERR_SEQ_LEN = -7,       /* device: seq_len < 0 or > pt_stride * page_size */
  MLRA_ERR_SCRATCH_LIMIT = -8, /* mlra_decode_noalloc: batch too large for its fixed scratch */
  MLRA_ERR_DRAIN = -9          /* device: after a wait timed out, copies or MMAs still in flight
                                  did not finish within the limit either, so shared memory or
                                  tensor memory may have been released under them. The CUDA
                                  context may be unusable: stop using it (and the process's
                                  device state) after this code. Overrides any other code. */
} mlra_status;

typedef enum { MLRA_F32 = 0, MLRA_BF16 = 1 } mlra_dtype;

/* Problem dimensions, in the pages' notation. */
typedef struct {
  int h;               /* query heads */
  int d_h;             /* head dim (width of q^C_h, K_h, V_h, o_h) */
  int d_c;             /* latent width over all k blocks */
  int d_rope;          /* decoupled RoPE key width d_h^R */
  int k;               /* latent blocks; 1 = MLA. k must divide d_c and h */
  int page_size;       /* tokens per cache page; must be 64 */
  float softmax_scale; /* <= 0 selects 1/sqrt(d_h + d_rope) (a reading: the pages fix none) */
  int blocks_summed;   /* 0: head group j = heads [j*h/k, (j+1)*h/k) attends only to block c_j
                          (the default reading). 1: every head attends to every block with its
                          own W^UK_{j,h}, W^UV_{j,h}, each block under its own softmax, and
                          o_h = attn_scale * sum_j W^UV_{j,h} o~_{j,h} (the reading Table 2 and
                          the alpha_attn entries of the MLRA index page's model tables point
                          to). Weights are then [k][h][d_b][d_h] and lse is [batch][k*h],
                          block-major (entry j*h + head). */
  float attn_scale;    /* alpha_attn when blocks_summed: <= 0 selects 1/sqrt(k), the values the
                          MLRA index page's appendix model tables print for MLRA-2 (sqrt(2)/2)
                          and MLRA-4 (1/2). Ignored otherwise. */
  int cache_fp8;       /* 0: bf16 cache. 1: E4M3 cache (the lesty.tech MLA article, section 5:
                          FP8 storage of the cached latent): every element of a cached row
                          [c | k^R] is one OCP E4M3 byte; the pool is then uint8
                          [num_pages][page_size][d_c + d_rope]. */
  float latent_scale;  /* E4M3 cache: value of a latent byte = latent_scale * e4m3(byte);
                          <= 0 selects 1. Ignored for a bf16 cache. */
  float rope_scale;    /* E4M3 cache: value of a RoPE-key byte = rope_scale * e4m3(byte);
                          <= 0 selects 1. Ignored for a bf16 cache. */
} mlra_config;

/* Compiled dims (others return MLRA_ERR_UNSUPPORTED), as (d_c/k, d_rope, heads per block, d_h),
 * heads per block being h/k, or h when blocks_summed:
 *   (32, 16, <=16, 32), (128, 64, <=32 or a multiple of 32, 128),
 *   (256, 64, <=64 or a multiple of 64, 128), (512, 64, <=64 or a multiple of 64, 128);
 * blocks_summed with k = 4 and (32, 16, ...) or (128, 64, ...), or k = 2 and (256, 64, ...);
 * cache_fp8 with (128, 64, a multiple of 32, 128) and blocks_summed = 0; batch <= 4096. */

typedef struct mlra_ctx* mlra_handle;

/* Creates a handle. w_uk, w_uv: device bf16 [h][d_c/k][d_h], row-major: W^UK_h maps a
 * block latent to a key by K_h[d] = sum_c c[c] * w_uk[h][c][d] (the ai360xpert code's
 * (H, d_c, d_head) convention restricted to the head's block); likewise w_uv for values.
 * With blocks_summed they are [k][h][d_c/k][d_h], one pair of matrices per block and head.
 * Borrowed, must stay valid and unchanged until mlra_destroy. *out receives the handle. */
int mlra_create(const mlra_config* cfg, const void* w_uk, const void* w_uv, mlra_handle* out);

/* Releases the handle (host memory only). NULL-safe. */
void mlra_destroy(mlra_handle h);

/* Bytes of device workspace mlra_decode needs for `batch` sequences (host output). */
int mlra_workspace_size(mlra_handle h, int batch, size_t* bytes);

/* One decode step for `batch` sequences.
 *   q          device [batch][h][d_h + d_rope], q^C_h then q^R_h (already rotated),
 *              dtype q_dtype (F32 or BF16; converted to bf16 for the tensor cores).
 *   pool       device bf16 [num_pages][page_size][d_c + d_rope]: token row = [c_1..c_k | k^R]
 *              (uint8 E4M3 bytes of the same shape when the handle has cache_fp8).
 *              16-byte aligned. Slots past a sequence's length may hold anything.
 *   page_table device int32 [batch][pt_stride]: token t of sequence b lives in slot
 *              t % page_size of page page_table[b*pt_stride + t/page_size].
 *   seq_lens   device int32 [batch], 0 <= n_b <= pt_stride * page_size. n_b = 0 gives
 *              o = 0 and lse = -inf.
 *   out        device [batch][h][d_h], dtype out_dtype.
 *   lse        device fp32 [batch][h] natural-log log-sum-exp of the scaled scores, or NULL.
 *   workspace  device, >= mlra_workspace_size(batch) bytes, 256-byte aligned. Its first
 *              4 bytes become this call's status word (the first kernel clears it once the
 *              kernel before it in the stream has finished); the next 16 bytes take errors
 *              found before that clear, which a later kernel of the call folds into it.
 * Launches three kernels on `stream`: query absorption, split-KV latent attention, and
 * log-sum-exp combine fused with the W^UV up-projection. All three use programmatic
 * dependent launch: the first may begin loading W^UK and setting up while the kernel before
 * it on `stream` finishes, and reads q (and writes the workspace) only after that kernel has
 * completed; stream order is otherwise unchanged. */
int mlra_decode(mlra_handle h, const void* q, mlra_dtype q_dtype, const void* pool,
                int num_pages, const int32_t* page_table, int pt_stride,
                const int32_t* seq_lens, int batch, void* out, mlra_dtype out_dtype,
                float* lse, void* workspace, size_t ws_bytes, void* stream);

/* mlra_decode for callers that cannot allocate device memory when they decode (a serving
 * engine whose KV-cache pool took all HBM left after the weights, a plug-in inside a runtime
 * that owns every allocation): no workspace argument, and nothing is allocated. The papers
 * have no counterpart: this is a property of the library, not of the method.
 *   Scratch: one 16 MiB device array inside the library (a static __device__ object), held
 *     by every GPU that loads the library until the process exits. Enough for
 *     mlra_workspace_size(batch) <= 16 MiB, i.e. MLRA-4 with 128 heads up to batch 124 on 148 SMs;
 *     larger requests return MLRA_ERR_SCRATCH_LIMIT before any launch.
 *   First call on a device: looks up the array's device address (cudaGetSymbolAddress) with
 *     that device current and keeps it. Make that first call before any stream capture. The
 *     address belongs to the device's current CUDA context: after that context is destroyed
 *     (cudaDeviceReset, for one) the kept address is stale, so a process that resets a device
 *     must not call this entry point again on it.
 *   Sharing: every call on a device uses the same array, which keeps the last call's
 *     contents; each call clears the status word it needs at zero. Calls whose kernels
 *     overlap on the GPU (other streams, threads or handles) race on the array: serialise
 *     them.
 *   status: device int32 word, or NULL. Receives this call's device status (0 = OK, else an
 *     mlra_status code) once the kernels have finished, in stream order. With NULL, device
 *     errors of this call are not reported.
 * All other arguments, layouts and results are those of mlra_decode. */
int mlra_decode_noalloc(mlra_handle h, const void* q, mlra_dtype q_dtype, const void* pool,
                        int num_pages, const int32_t* page_table, int pt_stride,
                        const int32_t* seq_lens, int batch, void* out, mlra_dtype out_dtype,
                        float* lse, int32_t* status, void* stream);

/* Same as mlra_decode but stops before the up-projection: latent_out receives the
 * normalised latent output o~ as device fp32 [batch][h][d_c/k], lse as above (nullable).
 * For testing the attention and indexing stages on their own. */
int mlra_decode_latent(mlra_handle h, const void* q, mlra_dtype q_dtype, const void* pool,
                       int num_pages, const int32_t* page_table, int pt_stride,
                       const int32_t* seq_lens, int batch, float* latent_out, float* lse,
                       void* workspace, size_t ws_bytes, void* stream);

/* mlra_decode for profiling: records events[0..3] (cudaEvent_t, created by the caller) on
 * `stream` before the absorb kernel, between the kernels and after the last one, and
 * launches without programmatic overlap so each event interval is one kernel's own time.
 * Results are identical to mlra_decode. */
int mlra_decode_profiled(mlra_handle h, const void* q, mlra_dtype q_dtype, const void* pool,
                         int num_pages, const int32_t* page_table, int pt_stride,
                         const int32_t* seq_lens, int batch, void* out, mlra_dtype out_dtype,
                         float* lse, void* workspace, size_t ws_bytes, void* const* events,
                         void* stream);

/* Writes new cache rows: token i goes to sequence seq_ids[i] at position positions[i], i.e.
 * slot positions[i] % page_size of page page_table[seq_ids[i]*pt_stride + positions[i]/page_size].
 *   c_new   device [n_tokens][d_c], kr_new device [n_tokens][d_rope], dtype in_dtype;
 *           F32 input is rounded to bf16 to nearest-even. With an E4M3 cache (cache_fp8) each
 *           element v is stored as the E4M3 byte nearest to v / scale (the quotient in fp32;
 *           ties to even; saturated at +-448), scale being latent_scale for c_new and
 *           rope_scale for kr_new.
 *   page_table has `batch` rows of pt_stride entries; seq_ids[i] must be < batch.
 *   status  device int32 word that receives a device error code (first error wins), or NULL.
 * Rows whose page id falls outside [0, num_pages), or whose sequence / position falls outside
 * the page table, are skipped and reported (MLRA_ERR_PAGE_OOB / MLRA_ERR_SEQ_LEN). */
int mlra_append_cache(mlra_handle h, void* pool, int num_pages, const int32_t* page_table,
                      int pt_stride, int batch, const int32_t* seq_ids, const int32_t* positions,
                      const void* c_new, const void* kr_new, mlra_dtype in_dtype,
                      int n_tokens, int32_t* status, void* stream);

/* Bytes of device workspace mlra_project_append needs (host output). d_model must be a
 * multiple of 128. */
int mlra_project_workspace_size(mlra_handle h, int batch, int d_model, size_t* bytes);

/* The step before decoding: computes each sequence's new cache row and stores it.
 * For token b with hidden state x[b] at position positions[b] (0-based index in its sequence):
 *   c   = x[b] W^DKV       (d_c latent features, all k blocks; the down-projection that the
 *                           "Multi-Head Low-Rank Attention: Making Compressed Attention Actually
 *                           Parallelizable" page's Core Mechanism and the lesty.tech MLA
 *                           article's section 4 describe)
 *   k^R = RoPE(x[b] W^KR)  (d_rope features; feature pair (2i, 2i+1) rotated by the angle
 *                           pos * rope_base^(-2i/d_rope), RoFormer's rotation, which the pages
 *                           cite but do not spell out)
 * and writes the bf16 (round to nearest even) row [c | k^R] into slot pos % page_size of page
 * page_table[b*pt_stride + pos/page_size]; with an E4M3 cache, the bytes e4m3(v / scale) as in
 * mlra_append_cache.
 *   x          device bf16 [batch][d_model], 16-byte aligned; d_model a multiple of 128.
 *   w_down     device bf16 [d_c + d_rope][d_model], 16-byte aligned: row r holds the weights
 *              of output feature r (the d_c latent features, then the d_rope RoPE-key
 *              features), i.e. W^DKV and W^KR transposed and stacked. Borrowed for the call.
 *   rope_base  RoPE base; <= 1 selects 10000.
 *   positions  device int32 [batch]; 0 <= pos < pt_stride * page_size, else the row is not
 *              written and the status word reads MLRA_ERR_SEQ_LEN.
 *   pool, num_pages, page_table, pt_stride: as in mlra_decode; a page id outside
 *              [0, num_pages) leaves the row unwritten and reports MLRA_ERR_PAGE_OOB.
 *   workspace  device, >= mlra_project_workspace_size bytes, 256-byte aligned; its first 4
 *              bytes become this call's status word (read it with mlra_get_status).
 * Launches two kernels on `stream` (a split-d_model tcgen05 GEMM into fp32 partials, then the
 * sum / rotation / store), both under programmatic dependent launch: the first loads W^DKV
 * while the previous kernel on `stream` finishes and reads x only after it has completed.
 * Rows of one call must go to distinct slots. */
int mlra_project_append(mlra_handle h, const void* x, int d_model, const void* w_down, float rope_base,
                        const int32_t* positions, void* pool, int num_pages, const int32_t* page_table,
                        int pt_stride, int batch, void* workspace, size_t ws_bytes, void* stream);

/* Runs the device split planner on seq_lens and writes the segments it would process:
 * segments device int32 [max_segments][5] rows (b, group, tile_begin, tile_end, slot),
 * count device int32. A group is a set of CTAs that shares one run of 128-token tiles;
 * the rule is documented in mlra_get_info's comment. For bit-exact tests of the plan. */
int mlra_plan(mlra_handle h, const int32_t* seq_lens, int batch, int pt_stride,
              int32_t* segments, int max_segments, int32_t* count, void* stream);

typedef struct {
  int num_sms;         /* SMs of the handle's device */
  int groups;          /* CTA groups of the decode kernel (floor(num_sms / ctas_per_group)) */
  int ctas_per_group;  /* one CTA per (latent block, head chunk) */
  int heads_per_cta;   /* query heads one CTA serves (padded to the MMA width) */
  int tile_tokens;     /* 128: split granularity. Plan rule: tiles_b = ceil(n_b/128),
                          T = sum tiles_b, quota = ceil(T/groups), group g takes flattened
                          tiles [g*quota, min((g+1)*quota, T)), partial slot = b + g. */
  int stages;          /* shared-memory pipeline depth of the decode kernel */
  float softmax_scale; /* the scale in use */
} mlra_info;

int mlra_get_info(mlra_handle h, mlra_info* out);

/* Copies a device status word (the first 4 bytes of a decode workspace, or an append status
 * word) to *out (host). Synchronous: call after the stream that wrote it has finished. */
int mlra_get_status(const void* status_word, int* out);

/* Static string for a status code. */
const char* mlra_status_string(int code);

#ifdef __cplusplus
}
#endif

#endif /* MLRA_H_ */
