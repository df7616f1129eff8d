// mlra_api.cu - the C ABI declared in include/mlra.h: argument checks, workspace carving,
// TMA tensor maps, and the launch sequence of one decode step
//   absorb (q -> packed absorbed query)  ->  latent attention (split-KV, persistent)
//   ->  combine + W^UV up-projection,
// chained with programmatic dependent launch so each kernel's prologue (barrier set-up,
// TMEM allocation, weight prefetch, split planning) overlaps the previous kernel's tail.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <atomic>
#include <cstring>
#include <mutex>

#include "../../include/mlra.h"
#include "aux_kernels.cuh"
#include "common.cuh"
#include "producer.cuh"
#include "decode.cuh"
#include "proj.cuh"

using namespace mlra;

namespace {

// ---------------------------------------------------------------------------------------
// Compiled kernel set. A variant fixes (d_b, d_rope, heads per CTA, d_h) and the decode
// kernel's shared-memory pipeline.
// ---------------------------------------------------------------------------------------
enum Variant { kTiny = 0, kMlra4 = 1, kMlra2 = 2, kMla = 3, kMlra4Sum = 4, kMlra2Sum = 5, kMlra4F8 = 6, kNumVariants };

using DecTiny = DecodeShape<32, 16, 16, 4, 2, 2>;
// P is written over each stage's RoPE columns, which leaves room for two query buffers (the
// next segment's query loads while the current one is in use)
using DecMlra4 = DecodeShape<128, 64, 32, 4, 2, 0>;
// MLRA-2 (and summed MLRA-2): two 80 KB stages beside the 40 KB query; P is written over each
// stage's RoPE columns, so the next tile's softmax does not wait for this tile's P.C
using DecMlra2 = DecodeShape<256, 64, 64, 2, 1, 0>;
// MLA (k = 1): a 128-token stage of whole 1152-byte rows is 144 KB, so one stage fits; 64
// heads per CTA (2 CTAs per group) halve the MMA work per cached byte against 32, and P goes
// into the stage so the 72 KB query fits beside it
using DecMla = DecodeShape<512, 64, 64, 1, 1, 0>;
// MLRA-4 with summed blocks: all h heads attend to each block, so a CTA takes 64 heads (an
// MMA of N = 64 costs the same issue time as N = 32); P lives in each stage's RoPE region so
// that four 48 KB stages fit next to the 24 KB query
using DecMlra4Sum = DecodeShape<128, 64, 64, 4, 1, 0>;
// MLRA-4 over an E4M3 cache: a 128-token tile is 24 KB (128-byte block rows, 64-byte RoPE
// rows), so eight fit beside two 12 KB query buffers (hi and lo terms of 32 heads), loaded and
// freed two tiles per barrier phase (four stages); three S buffers
using DecMlra4F8 = DecodeShape<128, 64, 32, 4, 2, 0, 3, true, 2, 2>;

constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // 1 s

struct VariantDims {
  int d_b, d_r, np, d_h;
};
constexpr VariantDims kDims[kNumVariants] = {
    {32, 16, 16, 32}, {128, 64, 32, 128}, {256, 64, 64, 128}, {512, 64, 64, 128}, {128, 64, 64, 128},
    {256, 64, 64, 128}, {128, 64, 32, 128}};

// Largest batch tile of the projection kernels: at d_b = 512 a 128-row tile of the merged
// latent plus W^UV^T would need 256 KB of shared memory.
template <int DB>
constexpr int max_nt() {
  return DB >= 512 ? 64 : 128;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

CUtensorMapSwizzle swizzle_for(int row_bytes) {
  return row_bytes == 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                          : row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_32B;
}

// 2-D tensor [rows][cols] of bf16 (esize 2) or bytes (esize 1), row stride in bytes, box
// [box_rows][box_cols], swizzled by the box's row width.
bool make_map(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t row_stride,
              uint32_t box_rows, uint32_t box_cols, int esize = 2) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_stride};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, esize == 1 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                  const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  swizzle_for(box_cols * esize), CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 3-D bf16 map over the query [batch][heads][cols]: box = cols x 1 head x box_b batch rows,
// landing as box_b rows of box_cols in shared memory.
bool make_q_map(CUtensorMap* m, const void* q, uint64_t batch, uint64_t heads, uint64_t cols, uint32_t box_cols,
                uint32_t box_b, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = get_encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {cols, heads, batch};
  cuuint64_t strides[2] = {cols * 2, heads * cols * 2};
  cuuint32_t box[3] = {box_cols, 1, box_b};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(q), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// A number unique to each host call that launches kernels (never 0): see EarlyTags.
std::atomic<unsigned> g_call_tag{0};
unsigned next_call_tag() {
  unsigned t = ++g_call_tag;
  while (t == 0) t = ++g_call_tag;
  return t;
}

int nt_for(int batch, int max_nt) {
  const int nt = batch <= 16 ? 16 : batch <= 32 ? 32 : batch <= 64 ? 64 : 128;
  return nt < max_nt ? nt : max_nt;
}

}  // namespace

struct mlra_ctx {
  mlra_config cfg;
  const void* w_uk;
  const void* w_uv;
  int device;
  int num_sms;
  Variant var;
  int d_b, d_r, np, chunks, nsub, heads_block, groups, stages;
  int vh;         // heads of the packed query and partials: h, or k*h when the blocks are summed
  bool summed;    // every head attends to every block; outputs summed
  float alpha;    // alpha_attn (summed blocks)
  bool fp8;       // E4M3 cache
  float latent_scale, rope_scale;
  float scale;
  CUtensorMap map_wuk;
  CUtensorMap map_wuv;
};

namespace {

// ----- per-variant launch helpers -----
// Every kernel asks for the largest shared-memory carve-out, so consecutive kernels of a step
// never make an SM switch its L1 / shared-memory split between them.
template <class K>
cudaError_t prep_kernel(K kernel, int smem) {
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributePreferredSharedMemoryCarveout,
                              cudaSharedmemCarveoutMaxShared);
}
cudaError_t prep_producer() {
  cudaError_t e = prep_kernel(mlra_down_proj_kernel<DownShape<16>>, DownShape<16>::SMEM);
  if (e == cudaSuccess) e = prep_kernel(mlra_down_proj_kernel<DownShape<32>>, DownShape<32>::SMEM);
  if (e == cudaSuccess) e = prep_kernel(mlra_down_proj_kernel<DownShape<64>>, DownShape<64>::SMEM);
  if (e == cudaSuccess) e = prep_kernel(mlra_down_proj_kernel<DownShape<128>>, DownShape<128>::SMEM);
  return e;
}

template <class Dec>
cudaError_t prep_decode() {
  return prep_kernel(mlra_decode_kernel<Dec>, Dec::SMEM_BYTES);
}
template <int DB, int DH, int NT>
cudaError_t prep_proj() {
  using S = ProjShape<DB, DH, NT>;
  cudaError_t e = prep_kernel(mlra_absorb_kernel<S>, S::SMEM1);
  if constexpr (DB == 128 && DH == 128)
    if (e == cudaSuccess) e = prep_kernel(mlra_absorb_kernel<S, true>, S::SMEM1F8);
  if (e != cudaSuccess) return e;
  e = prep_kernel(mlra_uproj_kernel<S, false>, S::SMEM4);
  if (e != cudaSuccess) return e;
  return prep_kernel(mlra_uproj_kernel<S, true>, S::SMEM4);
}
// combine + up-projection over SUMK summed blocks
template <int DB, int DH, int SUMK>
cudaError_t prep_proj_sum() {
  cudaError_t e;
  if ((e = prep_kernel(mlra_uproj_kernel<ProjShape<DB, DH, 16>, false, SUMK>, ProjShape<DB, DH, 16>::SMEM4)) !=
      cudaSuccess)
    return e;
  if ((e = prep_kernel(mlra_uproj_kernel<ProjShape<DB, DH, 32>, false, SUMK>, ProjShape<DB, DH, 32>::SMEM4)) !=
      cudaSuccess)
    return e;
  if ((e = prep_kernel(mlra_uproj_kernel<ProjShape<DB, DH, 64>, false, SUMK>, ProjShape<DB, DH, 64>::SMEM4)) !=
      cudaSuccess)
    return e;
  if constexpr (max_nt<DB>() >= 128)
    return prep_kernel(mlra_uproj_kernel<ProjShape<DB, DH, 128>, false, SUMK>, ProjShape<DB, DH, 128>::SMEM4);
  return cudaSuccess;
}
template <int DB, int DH>
cudaError_t prep_proj_all() {
  cudaError_t e;
  if ((e = prep_proj<DB, DH, 16>()) != cudaSuccess) return e;
  if ((e = prep_proj<DB, DH, 32>()) != cudaSuccess) return e;
  if ((e = prep_proj<DB, DH, 64>()) != cudaSuccess) return e;
  if constexpr (max_nt<DB>() >= 128) return prep_proj<DB, DH, 128>();
  return cudaSuccess;
}

// Programmatic dependent launch is on except inside a profiled call (thread-local, so a
// profiled call on one thread does not change another thread's launches).
thread_local bool g_use_pdl = true;

// `attr` must outlive the launch call that uses the returned config.
cudaLaunchConfig_t launch_cfg(dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                              cudaLaunchAttribute* attr) {
  cudaLaunchConfig_t c = {};
  c.gridDim = grid;
  c.blockDim = block;
  c.dynamicSmemBytes = smem;
  c.stream = s;
  if (pdl && g_use_pdl) {
    attr->id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr->val.programmaticStreamSerializationAllowed = 1;
    c.attrs = attr;
    c.numAttrs = 1;
  }
  return c;
}

template <int DB, int DH, int NT, bool F8 = false>
cudaError_t launch_absorb(const mlra_ctx* h, const ProjParams& pp, int batch, cudaStream_t s) {
  using S = ProjShape<DB, DH, NT>;
  // a bf16 query is read by TMA: its q^C columns in swizzle-width boxes, its q^R columns in one
  // unswizzled box
  CUtensorMap mqc, mqr;
  std::memset(&mqc, 0, sizeof(mqc));
  std::memset(&mqr, 0, sizeof(mqr));
  if (!pp.q_f32) {
    const uint64_t cols = (uint64_t)DH + h->d_r;
    if (!make_q_map(&mqc, pp.q, batch, h->cfg.h, cols, S::AW, NT, swizzle_for(S::AROWB)) ||
        !make_q_map(&mqr, pp.q, batch, h->cfg.h, cols, h->d_r, NT, CU_TENSOR_MAP_SWIZZLE_NONE))
      return cudaErrorInvalidValue;
  }
  cudaLaunchAttribute attr;
  cudaLaunchConfig_t c = launch_cfg(dim3(h->vh, (batch + NT - 1) / NT), dim3(kProjThreads),
                                    F8 ? S::SMEM1F8 : S::SMEM1, s, true, &attr);
  return cudaLaunchKernelEx(&c, mlra_absorb_kernel<S, F8>, h->map_wuk, mqc, mqr, pp);
}
template <int DB, int DH, int NT, bool LATENT, int SUMK = 1>
cudaError_t launch_uproj(const mlra_ctx* h, const ProjParams& pp, int batch, cudaStream_t s) {
  using S = ProjShape<DB, DH, NT>;
  // one CTA per output head; per virtual head when only the latent is wanted
  const int gx = SUMK > 1 ? h->cfg.h : h->vh;
  cudaLaunchAttribute attr;
  cudaLaunchConfig_t c = launch_cfg(dim3(gx, (batch + NT - 1) / NT), dim3(kProjThreads), S::SMEM4, s, true,
                                    &attr);
  return cudaLaunchKernelEx(&c, mlra_uproj_kernel<S, LATENT, SUMK>, h->map_wuv, pp);
}
template <int DB, int DH, bool F8 = false>
cudaError_t dispatch_absorb(const mlra_ctx* h, const ProjParams& pp, int batch, cudaStream_t s) {
  switch (nt_for(batch, max_nt<DB>())) {
    case 16: return launch_absorb<DB, DH, 16, F8>(h, pp, batch, s);
    case 32: return launch_absorb<DB, DH, 32, F8>(h, pp, batch, s);
    case 64: return launch_absorb<DB, DH, 64, F8>(h, pp, batch, s);
    default:
      if constexpr (max_nt<DB>() >= 128) return launch_absorb<DB, DH, 128, F8>(h, pp, batch, s);
      return cudaErrorInvalidValue;
  }
}
template <int DB, int DH, bool LATENT, int SUMK = 1>
cudaError_t dispatch_uproj(const mlra_ctx* h, const ProjParams& pp, int batch, cudaStream_t s) {
  switch (nt_for(batch, max_nt<DB>())) {
    case 16: return launch_uproj<DB, DH, 16, LATENT, SUMK>(h, pp, batch, s);
    case 32: return launch_uproj<DB, DH, 32, LATENT, SUMK>(h, pp, batch, s);
    case 64: return launch_uproj<DB, DH, 64, LATENT, SUMK>(h, pp, batch, s);
    default:
      if constexpr (max_nt<DB>() >= 128) return launch_uproj<DB, DH, 128, LATENT, SUMK>(h, pp, batch, s);
      return cudaErrorInvalidValue;
  }
}

template <class Dec>
cudaError_t launch_decode(const mlra_ctx* h, const CUtensorMap& mc, const CUtensorMap& mr,
                          const CUtensorMap& mqc, const CUtensorMap& mqr, const DecodeParams& dp,
                          cudaStream_t s) {
  cudaLaunchAttribute attr;
  cudaLaunchConfig_t c = launch_cfg(dim3(h->groups * h->nsub), dim3(Dec::THREADS), Dec::SMEM_BYTES, s, true, &attr);
  return cudaLaunchKernelEx(&c, mlra_decode_kernel<Dec>, mc, mr, mqc, mqr, dp);
}

struct Workspace {
  int* status;
  __nv_bfloat16* q_pack;
  float* qfac;  // E4M3 cache only
  float* o_part;
  float* lse_part;
  size_t bytes;
};

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

Workspace carve(const mlra_ctx* h, int batch, void* base) {
  Workspace w;
  char* p = static_cast<char*>(base);
  size_t off = 0;
  w.status = reinterpret_cast<int*>(p + off);
  off += 256;
  w.q_pack = reinterpret_cast<__nv_bfloat16*>(p + off);
  // bf16 rows, or two E4M3 rows (the hi and lo terms) per head: the same bytes
  off += align256((size_t)batch * h->nsub * h->np * (h->d_b + h->d_r) * 2);
  w.qfac = nullptr;
  if (h->fp8) {
    w.qfac = reinterpret_cast<float*>(p + off);
    off += align256((size_t)batch * h->nsub * h->np * 4);
  }
  const size_t slots = (size_t)batch + h->groups;
  w.o_part = reinterpret_cast<float*>(p + off);
  off += align256(slots * h->vh * h->d_b * 4);
  w.lse_part = reinterpret_cast<float*>(p + off);
  off += align256(slots * h->vh * 4);
  w.bytes = off;
  return w;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int run_decode(mlra_handle h, const void* q, mlra_dtype q_dtype, const void* pool, int num_pages,
               const int32_t* page_table, int pt_stride, const int32_t* seq_lens, int batch, void* out,
               mlra_dtype out_dtype, float* lse, float* latent_out, void* workspace, size_t ws_bytes,
               void* stream, int inject_stall, unsigned long long wait_limit_ns,
               void* const* events = nullptr) {
  if (!h || !q || !pool || !page_table || !seq_lens || !workspace) return MLRA_ERR_INVALID_ARG;
  if (!out && !latent_out) return MLRA_ERR_INVALID_ARG;
  if (batch <= 0 || batch > 4096 || num_pages <= 0 || pt_stride <= 0) return MLRA_ERR_INVALID_ARG;
  if ((q_dtype != MLRA_F32 && q_dtype != MLRA_BF16) || (out && out_dtype != MLRA_F32 && out_dtype != MLRA_BF16))
    return MLRA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(pool) || (reinterpret_cast<uintptr_t>(workspace) & 255))
    return MLRA_ERR_INVALID_ARG;
  if ((long long)num_pages * kPage > 0x7fffffffLL) return MLRA_ERR_UNSUPPORTED;
  Workspace w = carve(h, batch, workspace);
  if (ws_bytes < w.bytes) return MLRA_ERR_WORKSPACE;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return MLRA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int D = h->cfg.d_c + h->d_r;

  // tensor maps over this call's pool and packed-query buffers; a box row is at most 128 bytes
  const int es = h->fp8 ? 1 : 2;  // bytes per cached / packed-query element
  const int cw = h->d_b * es < 128 ? h->d_b : 128 / es, rw = h->d_r * es < 128 ? h->d_r : 128 / es;
  const int nq = h->fp8 ? 2 : 1;  // query rows per head (E4M3: hi and lo terms)
  CUtensorMap mc, mr, mqc, mqr;
  const uint64_t qrows = (uint64_t)batch * h->nsub * h->np * nq;
  // a head chunk narrower than the MMA's N loads only its real rows (bf16 shapes only: the
  // E4M3 shape's hi and lo rows come as one box, so its chunks are always full)
  const uint32_t q_rows = h->heads_block < h->np ? h->heads_block : h->np;
  const uint64_t qw = h->d_b + h->d_r;
  if (!make_map(&mc, pool, (uint64_t)num_pages * kPage, D, (uint64_t)D * es, kPage, cw, es) ||
      !make_map(&mr, pool, (uint64_t)num_pages * kPage, D, (uint64_t)D * es, kPage, rw, es) ||
      !make_map(&mqc, w.q_pack, qrows, qw, qw * es, q_rows * nq, cw, es) ||
      !make_map(&mqr, w.q_pack, qrows, qw, qw * es, q_rows * nq, rw, es))
    return MLRA_ERR_CUDA;

  ProjParams pp = {};
  pp.q = q;
  pp.q_f32 = q_dtype == MLRA_F32;
  pp.q_pack = w.q_pack;
  pp.qscale = h->scale * kLog2e;
  pp.d_r = h->d_r;
  pp.np = h->np;
  pp.nsub = h->nsub;
  pp.chunks = h->chunks;
  pp.heads_block = h->heads_block;
  pp.o_part = w.o_part;
  pp.lse_part = w.lse_part;
  pp.out = out;
  pp.out_f32 = out_dtype == MLRA_F32;
  pp.lse_out = lse;
  pp.latent_out = latent_out;
  pp.seq_lens = seq_lens;
  pp.pt_stride = pt_stride;
  pp.groups = h->groups;
  pp.batch = batch;
  pp.h = h->vh;
  pp.q_heads = h->cfg.h;
  pp.out_heads = h->cfg.h;
  pp.out_scale = h->summed ? h->alpha : 1.f;
  pp.latent_scale = h->latent_scale;
  pp.rope_scale = h->rope_scale;
  pp.qfac = w.qfac;
  pp.q_rows_per_sub = h->np * nq;
  // the status word's first 4 bytes; the next two words take early errors by call tag
  const EarlyTags tags = {reinterpret_cast<unsigned*>(w.status) + 1, next_call_tag()};
  pp.status = w.status;
  pp.tags = tags;
  pp.wait_limit_ns = wait_limit_ns;
  pp.inject_stall = inject_stall;

  DecodeParams dp = {};
  dp.seq_lens = seq_lens;
  dp.page_table = page_table;
  dp.pt_stride = pt_stride;
  dp.batch = batch;
  dp.num_pages = num_pages;
  dp.groups = h->groups;
  dp.nsub = h->nsub;
  dp.chunks = h->chunks;
  dp.heads_block = h->heads_block;
  dp.h = h->vh;
  dp.d_c = h->cfg.d_c;
  dp.q_rows = (int)q_rows;
  dp.qfac = w.qfac;
  dp.o_scale = h->fp8 ? h->latent_scale / DecMlra4F8::P_SCALE : 1.f;
  dp.o_part = w.o_part;
  dp.lse_part = w.lse_part;
  dp.status = w.status;
  dp.tags = tags;
  dp.wait_limit_ns = wait_limit_ns;
  dp.inject_stall = inject_stall;

  cudaError_t e = cudaSuccess;
  const bool latent = latent_out != nullptr;
  // profiling: events between the kernels (and no programmatic overlap, so each interval
  // is one kernel's own time)
  const bool prof = events != nullptr;
  auto rec = [&](int i) {
    if (prof && e == cudaSuccess) e = cudaEventRecord(static_cast<cudaEvent_t>(events[i]), s);
  };
  g_use_pdl = !prof;
  rec(0);
  switch (h->var) {
    case kTiny:
      e = dispatch_absorb<32, 32>(h, pp, batch, s);
      rec(1);
      if (e == cudaSuccess) e = launch_decode<DecTiny>(h, mc, mr, mqc, mqr, dp, s);
      rec(2);
      if (e == cudaSuccess)
        e = latent      ? dispatch_uproj<32, 32, true>(h, pp, batch, s)
            : h->summed ? dispatch_uproj<128, 32, false, 4>(h, pp, batch, s)
                        : dispatch_uproj<32, 32, false>(h, pp, batch, s);
      break;
    case kMlra4:
      e = dispatch_absorb<128, 128>(h, pp, batch, s);
      rec(1);
      if (e == cudaSuccess)
        e = launch_decode<DecMlra4>(h, mc, mr, mqc, mqr, dp, s);
      rec(2);
      if (e == cudaSuccess)
        e = latent ? dispatch_uproj<128, 128, true>(h, pp, batch, s)
                   : dispatch_uproj<128, 128, false>(h, pp, batch, s);
      break;
    case kMlra4Sum:
      e = dispatch_absorb<128, 128>(h, pp, batch, s);
      rec(1);
      if (e == cudaSuccess) e = launch_decode<DecMlra4Sum>(h, mc, mr, mqc, mqr, dp, s);
      rec(2);
      if (e == cudaSuccess)
        e = latent ? dispatch_uproj<128, 128, true>(h, pp, batch, s)
                   : dispatch_uproj<512, 128, false, 4>(h, pp, batch, s);
      break;
    case kMlra2:
      e = dispatch_absorb<256, 128>(h, pp, batch, s);
      rec(1);
      if (e == cudaSuccess) e = launch_decode<DecMlra2>(h, mc, mr, mqc, mqr, dp, s);
      rec(2);
      if (e == cudaSuccess)
        e = latent ? dispatch_uproj<256, 128, true>(h, pp, batch, s)
                   : dispatch_uproj<256, 128, false>(h, pp, batch, s);
      break;
    case kMlra2Sum:
      // every head on each of the two 256-wide blocks: the MLRA-2 decode kernel over 2h
      // virtual heads, then one GEMM over the stacked 512-wide merged latents
      e = dispatch_absorb<256, 128>(h, pp, batch, s);
      rec(1);
      if (e == cudaSuccess) e = launch_decode<DecMlra2>(h, mc, mr, mqc, mqr, dp, s);
      rec(2);
      if (e == cudaSuccess)
        e = latent ? dispatch_uproj<256, 128, true>(h, pp, batch, s)
                   : dispatch_uproj<512, 128, false, 2>(h, pp, batch, s);
      break;
    case kMlra4F8:
      e = dispatch_absorb<128, 128, true>(h, pp, batch, s);
      rec(1);
      if (e == cudaSuccess) e = launch_decode<DecMlra4F8>(h, mc, mr, mqc, mqr, dp, s);
      rec(2);
      if (e == cudaSuccess)
        e = latent ? dispatch_uproj<128, 128, true>(h, pp, batch, s)
                   : dispatch_uproj<128, 128, false>(h, pp, batch, s);
      break;
    case kMla:
      e = dispatch_absorb<512, 128>(h, pp, batch, s);
      rec(1);
      if (e == cudaSuccess) e = launch_decode<DecMla>(h, mc, mr, mqc, mqr, dp, s);
      rec(2);
      if (e == cudaSuccess)
        e = latent ? dispatch_uproj<512, 128, true>(h, pp, batch, s)
                   : dispatch_uproj<512, 128, false>(h, pp, batch, s);
      break;
    default:
      return MLRA_ERR_UNSUPPORTED;
  }
  rec(3);
  g_use_pdl = true;
  return e == cudaSuccess ? MLRA_OK : MLRA_ERR_CUDA;
}

// ---------------------------------------------------------------------------------------
// Scratch of mlra_decode_noalloc: mlra_decode with its workspace in a fixed device array of
// this library instead of one the caller passes. It exists for callers that cannot allocate
// device memory at the point where they decode: a serving engine that has handed all free
// HBM to its KV-cache page pool once the weights were loaded (a per-step allocation would
// fail, or would force the pool to shrink), or a plug-in that runs inside another runtime
// which owns every allocation and hands it only the tensors of the step.
//
// kNoAllocScratchBytes is the whole array; every GPU that loads this library holds it until
// the process exits. It covers mlra_workspace_size(batch) for MLRA-4 with 128 heads up to
// batch 124 on a 148-SM GPU. All calls on a device share the one array and it keeps what the
// last call left there: the status word is cleared by the call's first kernel, as in
// mlra_decode, and every other byte the kernels read is written earlier in the same call. Calls whose kernels overlap on the GPU (other
// streams, other threads, other handles on the same device) race on it.
// ---------------------------------------------------------------------------------------
constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};

// Device address of g_noalloc_scratch on `dev`, which must be the current device. In host
// code the array's name only identifies the symbol; the address is looked up once per device
// (the first mlra_decode_noalloc call there) and kept.
int noalloc_scratch(int dev, void** out) {
  if (dev < 0 || dev >= kNoAllocMaxDevices) return MLRA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* ptr = nullptr;
    if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) {
      cudaGetLastError();
      return MLRA_ERR_CUDA;
    }
    g_noalloc_ptr[dev] = ptr;
  }
  *out = g_noalloc_ptr[dev];
  return MLRA_OK;
}

}  // namespace

namespace {
constexpr int kProjSlice = 128;  // d_model columns per down-projection CTA
size_t project_ws_bytes(const mlra_ctx* h, int batch, int d_model) {
  const size_t d_out = (size_t)h->cfg.d_c + h->d_r;
  return 256 + ((size_t)(d_model / kProjSlice) * batch * d_out * 4 + 255) / 256 * 256;
}
template <int NT>
cudaError_t launch_down_proj(const CUtensorMap& mw, const CUtensorMap& mx, const DownParams& dp, int d_out,
                             int kslices, int batch, cudaStream_t s) {
  using S = DownShape<NT>;
  cudaLaunchAttribute attr;
  cudaLaunchConfig_t c = launch_cfg(dim3((d_out + 127) / 128, kslices, (batch + NT - 1) / NT), dim3(S::THREADS),
                                    S::SMEM, s, true, &attr);
  return cudaLaunchKernelEx(&c, mlra_down_proj_kernel<S>, mw, mx, dp);
}
}  // namespace

extern "C" {

int mlra_create(const mlra_config* cfg, const void* w_uk, const void* w_uv, mlra_handle* out) {
  if (!cfg || !w_uk || !w_uv || !out) return MLRA_ERR_INVALID_ARG;
  *out = nullptr;
  const mlra_config& c = *cfg;
  if (c.h <= 0 || c.d_h <= 0 || c.d_c <= 0 || c.d_rope <= 0 || c.k <= 0) return MLRA_ERR_INVALID_ARG;
  if (c.d_c % c.k != 0 || c.h % c.k != 0) return MLRA_ERR_INVALID_ARG;
  if (c.page_size != kPage) return MLRA_ERR_UNSUPPORTED;
  if (!aligned16(w_uk) || !aligned16(w_uv)) return MLRA_ERR_INVALID_ARG;
  if (c.blocks_summed != 0 && c.blocks_summed != 1) return MLRA_ERR_INVALID_ARG;
  const bool summed = c.blocks_summed == 1;
  // heads per block: a group of h/k, or all h when every head attends to every block
  const int d_b = c.d_c / c.k, hb = summed ? c.h : c.h / c.k;
  int var = -1;
  for (int v = 0; v < kMlra4Sum; ++v)  // the summed-only shapes are chosen below
    if (kDims[v].d_b == d_b && kDims[v].d_r == c.d_rope && kDims[v].d_h == c.d_h &&
        (hb <= kDims[v].np || hb % kDims[v].np == 0))
      var = v;
  if (var < 0) return MLRA_ERR_UNSUPPORTED;
  // summed blocks: the combine's GEMM runs over k*d_b, compiled for these three shapes
  if (summed && !((var == kMlra4 && c.k == 4) || (var == kTiny && c.k == 4) || (var == kMlra2 && c.k == 2)))
    return MLRA_ERR_UNSUPPORTED;
  if (summed && var == kMlra4) var = kMlra4Sum;
  if (summed && var == kMlra2) var = kMlra2Sum;
  // E4M3 cache: compiled for the MLRA-4 block shape (d_b 128, d_rope 64, d_h 128), partitioned
  // heads, whole 32-head chunks
  if (c.cache_fp8 != 0 && c.cache_fp8 != 1) return MLRA_ERR_INVALID_ARG;
  const bool fp8 = c.cache_fp8 == 1;
  if (fp8 && (summed || var != kMlra4 || hb % 32 != 0)) return MLRA_ERR_UNSUPPORTED;
  if (fp8 && (!(c.latent_scale >= 0.f) || !(c.rope_scale >= 0.f) || !std::isfinite(c.latent_scale) ||
              !std::isfinite(c.rope_scale)))
    return MLRA_ERR_INVALID_ARG;
  if (fp8) var = kMlra4F8;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return MLRA_ERR_CUDA;
  cudaDeviceProp prop;
  if (cudaGetDeviceProperties(&prop, dev) != cudaSuccess) return MLRA_ERR_CUDA;
  if (prop.major != 10) return MLRA_ERR_UNSUPPORTED;

  mlra_ctx* h = new mlra_ctx();
  h->cfg = c;
  h->w_uk = w_uk;
  h->w_uv = w_uv;
  h->device = dev;
  h->num_sms = prop.multiProcessorCount;
  h->var = static_cast<Variant>(var);
  h->d_b = d_b;
  h->d_r = c.d_rope;
  h->np = kDims[var].np;
  h->heads_block = hb;
  h->summed = summed;
  h->vh = summed ? c.k * c.h : c.h;
  h->alpha = c.attn_scale > 0.f ? c.attn_scale : 1.0f / sqrtf((float)c.k);
  h->fp8 = fp8;
  h->latent_scale = fp8 && c.latent_scale > 0.f ? c.latent_scale : 1.f;
  h->rope_scale = fp8 && c.rope_scale > 0.f ? c.rope_scale : 1.f;
  h->chunks = (hb + h->np - 1) / h->np;
  h->nsub = c.k * h->chunks;
  h->groups = h->num_sms / h->nsub;
  h->scale = c.softmax_scale > 0.f ? c.softmax_scale : 1.0f / std::sqrt((float)(c.d_h + c.d_rope));
  h->stages = 0;

  cudaError_t e = cudaSuccess;
  switch (h->var) {
    case kTiny:
      e = prep_decode<DecTiny>();
      if (e == cudaSuccess) e = prep_proj_all<32, 32>();
      if (e == cudaSuccess && summed) e = prep_proj_sum<128, 32, 4>();
      h->stages = DecTiny::STAGES;
      break;
    case kMlra4:
      e = prep_decode<DecMlra4>();
      if (e == cudaSuccess) e = prep_proj_all<128, 128>();
      h->stages = DecMlra4::STAGES;
      break;
    case kMlra4Sum:
      e = prep_decode<DecMlra4Sum>();
      if (e == cudaSuccess) e = prep_proj_all<128, 128>();
      if (e == cudaSuccess) e = prep_proj_sum<512, 128, 4>();
      h->stages = DecMlra4Sum::STAGES;
      break;
    case kMlra2:
      e = prep_decode<DecMlra2>();
      if (e == cudaSuccess) e = prep_proj_all<256, 128>();
      h->stages = DecMlra2::STAGES;
      break;
    case kMla:
      e = prep_decode<DecMla>();
      if (e == cudaSuccess) e = prep_proj_all<512, 128>();
      h->stages = DecMla::STAGES;
      break;
    case kMlra4F8:
      e = prep_decode<DecMlra4F8>();
      if (e == cudaSuccess) e = prep_proj_all<128, 128>();
      h->stages = DecMlra4F8::STAGES;
      break;
    case kMlra2Sum:
      e = prep_decode<DecMlra2>();
      if (e == cudaSuccess) e = prep_proj_all<256, 128>();
      if (e == cudaSuccess) e = prep_proj_sum<512, 128, 2>();
      h->stages = DecMlra2::STAGES;
      break;
    default:
      break;
  }
  if (e == cudaSuccess) e = prep_producer();
  if (e != cudaSuccess) {
    delete h;
    return MLRA_ERR_CUDA;
  }
  const int aw = c.d_h < 64 ? c.d_h : 64;
  const int nmt_rows = d_b >= 128 ? d_b : 128;
  const uint32_t boxr1 = nmt_rows < 256 ? nmt_rows : 256;
  const uint32_t boxr4 = d_b < 256 ? d_b : 256;
  // weight tensor maps: [vh * d_b rows][d_h cols], one d_b-row matrix per (virtual) head
  if (!make_map(&h->map_wuk, w_uk, (uint64_t)h->vh * d_b, c.d_h, (uint64_t)c.d_h * 2, boxr1, aw) ||
      !make_map(&h->map_wuv, w_uv, (uint64_t)h->vh * d_b, c.d_h, (uint64_t)c.d_h * 2, boxr4, aw)) {
    delete h;
    return MLRA_ERR_CUDA;
  }
  *out = h;
  return MLRA_OK;
}

void mlra_destroy(mlra_handle h) { delete h; }

int mlra_workspace_size(mlra_handle h, int batch, size_t* bytes) {
  if (!h || !bytes || batch <= 0 || batch > 4096) return MLRA_ERR_INVALID_ARG;
  *bytes = carve(h, batch, nullptr).bytes;
  return MLRA_OK;
}

int mlra_decode(mlra_handle h, const void* q, mlra_dtype q_dtype, const void* pool, int num_pages,
                const int32_t* page_table, int pt_stride, const int32_t* seq_lens, int batch, void* out,
                mlra_dtype out_dtype, float* lse, void* workspace, size_t ws_bytes, void* stream) {
  if (!out) return MLRA_ERR_INVALID_ARG;
  return run_decode(h, q, q_dtype, pool, num_pages, page_table, pt_stride, seq_lens, batch, out, out_dtype,
                    lse, nullptr, workspace, ws_bytes, stream, 0, kWaitLimitNs);
}

int mlra_decode_noalloc(mlra_handle h, const void* q, mlra_dtype q_dtype, const void* pool, int num_pages,
                        const int32_t* page_table, int pt_stride, const int32_t* seq_lens, int batch,
                        void* out, mlra_dtype out_dtype, float* lse, int32_t* status, void* stream) {
  if (!h || !out || batch <= 0 || batch > 4096) return MLRA_ERR_INVALID_ARG;
  if (carve(h, batch, nullptr).bytes > kNoAllocScratchBytes) return MLRA_ERR_SCRATCH_LIMIT;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return MLRA_ERR_INVALID_ARG;
  void* scratch = nullptr;
  int rc = noalloc_scratch(dev, &scratch);
  if (rc != MLRA_OK) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rc = run_decode(h, q, q_dtype, pool, num_pages, page_table, pt_stride, seq_lens, batch, out, out_dtype, lse,
                  nullptr, scratch, kNoAllocScratchBytes, stream, 0, kWaitLimitNs);
  if (rc != MLRA_OK) return rc;
  if (status && cudaMemcpyAsync(status, scratch, sizeof(int32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
    return MLRA_ERR_CUDA;
  return MLRA_OK;
}

int mlra_decode_latent(mlra_handle h, const void* q, mlra_dtype q_dtype, const void* pool, int num_pages,
                       const int32_t* page_table, int pt_stride, const int32_t* seq_lens, int batch,
                       float* latent_out, float* lse, void* workspace, size_t ws_bytes, void* stream) {
  if (!latent_out) return MLRA_ERR_INVALID_ARG;
  return run_decode(h, q, q_dtype, pool, num_pages, page_table, pt_stride, seq_lens, batch, nullptr,
                    MLRA_F32, lse, latent_out, workspace, ws_bytes, stream, 0, kWaitLimitNs);
}

int mlra_append_cache(mlra_handle h, void* pool, int num_pages, const int32_t* page_table, int pt_stride,
                      int batch, const int32_t* seq_ids, const int32_t* positions, const void* c_new,
                      const void* kr_new, mlra_dtype in_dtype, int n_tokens, int32_t* status, void* stream) {
  if (!h || !pool || !page_table || !seq_ids || !positions || !c_new || !kr_new) return MLRA_ERR_INVALID_ARG;
  if (n_tokens < 0 || num_pages <= 0 || pt_stride <= 0 || batch <= 0) return MLRA_ERR_INVALID_ARG;
  if (in_dtype != MLRA_F32 && in_dtype != MLRA_BF16) return MLRA_ERR_INVALID_ARG;
  if (n_tokens == 0) return MLRA_OK;
  const int warps = 8;
  if (h->fp8)
    mlra_append_e4m3_kernel<<<(n_tokens + warps - 1) / warps, warps * 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<uint8_t*>(pool), num_pages, page_table, pt_stride, batch, seq_ids, positions, c_new, kr_new,
        in_dtype == MLRA_F32, n_tokens, h->cfg.d_c, h->d_r, h->latent_scale, h->rope_scale, status);
  else
    mlra_append_kernel<<<(n_tokens + warps - 1) / warps, warps * 32, 0, static_cast<cudaStream_t>(stream)>>>(
        static_cast<__nv_bfloat16*>(pool), num_pages, page_table, pt_stride, batch, seq_ids, positions, c_new,
        kr_new, in_dtype == MLRA_F32, n_tokens, h->cfg.d_c, h->d_r, status);
  return cudaGetLastError() == cudaSuccess ? MLRA_OK : MLRA_ERR_CUDA;
}

int mlra_project_workspace_size(mlra_handle h, int batch, int d_model, size_t* bytes) {
  if (!h || !bytes || batch < 0 || d_model <= 0 || d_model % kProjSlice != 0) return MLRA_ERR_INVALID_ARG;
  *bytes = project_ws_bytes(h, batch, d_model);
  return MLRA_OK;
}

int mlra_project_append(mlra_handle h, const void* x, int d_model, const void* w_down, float rope_base,
                        const int32_t* positions, void* pool, int num_pages, const int32_t* page_table,
                        int pt_stride, int batch, void* workspace, size_t ws_bytes, void* stream) {
  if (!h || !x || !w_down || !positions || !pool || !page_table || !workspace) return MLRA_ERR_INVALID_ARG;
  if (batch < 0 || batch > 65536 || num_pages <= 0 || pt_stride <= 0) return MLRA_ERR_INVALID_ARG;
  if (d_model <= 0 || d_model % kProjSlice != 0) return MLRA_ERR_INVALID_ARG;
  const int d_out = h->cfg.d_c + h->d_r;
  if (d_out % 2 != 0 || h->d_r % 2 != 0) return MLRA_ERR_UNSUPPORTED;
  if (!aligned16(x) || !aligned16(w_down) || reinterpret_cast<uintptr_t>(workspace) % 256 != 0 ||
      reinterpret_cast<uintptr_t>(pool) % 4 != 0)
    return MLRA_ERR_INVALID_ARG;
  if (ws_bytes < project_ws_bytes(h, batch, d_model)) return MLRA_ERR_WORKSPACE;
  if (batch == 0) return MLRA_OK;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev != h->device) return MLRA_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  int* status = static_cast<int*>(workspace);
  g_use_pdl = true;
  const int nt = nt_for(batch, 128);
  const int kslices = d_model / kProjSlice;
  CUtensorMap mw, mx;
  if (!make_map(&mw, w_down, (uint64_t)d_out, (uint64_t)d_model, (uint64_t)d_model * 2, 128, 64) ||
      !make_map(&mx, x, (uint64_t)batch, (uint64_t)d_model, (uint64_t)d_model * 2, (uint32_t)nt, 64))
    return MLRA_ERR_CUDA;
  float* part = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + 256);
  const EarlyTags tags = {reinterpret_cast<unsigned*>(status) + 1, next_call_tag()};
  DownParams dp = {d_out, batch, part, status, tags, kWaitLimitNs};
  cudaError_t e;
  switch (nt) {
    case 16: e = launch_down_proj<16>(mw, mx, dp, d_out, kslices, batch, s); break;
    case 32: e = launch_down_proj<32>(mw, mx, dp, d_out, kslices, batch, s); break;
    case 64: e = launch_down_proj<64>(mw, mx, dp, d_out, kslices, batch, s); break;
    default: e = launch_down_proj<128>(mw, mx, dp, d_out, kslices, batch, s); break;
  }
  if (e != cudaSuccess) return MLRA_ERR_CUDA;
  AppendRowParams ap = {part, kslices, batch, h->cfg.d_c, h->d_r, d_out, positions, page_table, pt_stride,
                        num_pages, pool, h->fp8 ? 1 : 0, h->latent_scale, h->rope_scale,
                        std::log2((double)(rope_base > 1.f ? rope_base : 10000.f)), status, tags};
  const int total = batch * (d_out / 2);
  cudaLaunchAttribute attr;
  cudaLaunchConfig_t c = launch_cfg(dim3((total + kAppendPairs - 1) / kAppendPairs),
                                    dim3(kAppendPairs, kAppendGroups), 0, s, true, &attr);
  if (cudaLaunchKernelEx(&c, mlra_rope_append_kernel, ap) != cudaSuccess) return MLRA_ERR_CUDA;
  return MLRA_OK;
}

int mlra_plan(mlra_handle h, const int32_t* seq_lens, int batch, int pt_stride, int32_t* segments,
              int max_segments, int32_t* count, void* stream) {
  if (!h || !seq_lens || !segments || !count || batch <= 0 || max_segments < 0 || pt_stride <= 0)
    return MLRA_ERR_INVALID_ARG;
  mlra_plan_kernel<<<1, 192, 0, static_cast<cudaStream_t>(stream)>>>(seq_lens, batch, pt_stride, h->groups,
                                                                    segments, max_segments, count, nullptr);
  return cudaGetLastError() == cudaSuccess ? MLRA_OK : MLRA_ERR_CUDA;
}

int mlra_get_info(mlra_handle h, mlra_info* out) {
  if (!h || !out) return MLRA_ERR_INVALID_ARG;
  out->num_sms = h->num_sms;
  out->groups = h->groups;
  out->ctas_per_group = h->nsub;
  out->heads_per_cta = h->np;
  out->tile_tokens = kTile;
  out->stages = h->stages;
  out->softmax_scale = h->scale;
  return MLRA_OK;
}

int mlra_get_status(const void* status_word, int* out) {
  if (!status_word || !out) return MLRA_ERR_INVALID_ARG;
  int v = 0;
  if (cudaMemcpy(&v, status_word, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return MLRA_ERR_CUDA;
  *out = v;
  return MLRA_OK;
}

const char* mlra_status_string(int code) {
  switch (code) {
    case MLRA_OK: return "ok";
    case MLRA_ERR_INVALID_ARG: return "invalid argument";
    case MLRA_ERR_UNSUPPORTED: return "unsupported dimensions or device";
    case MLRA_ERR_CUDA: return "CUDA runtime error";
    case MLRA_ERR_PAGE_OOB: return "page id outside the pool";
    case MLRA_ERR_TIMEOUT: return "device pipeline wait timed out";
    case MLRA_ERR_WORKSPACE: return "workspace too small";
    case MLRA_ERR_SEQ_LEN: return "sequence length outside its page-table row";
    case MLRA_ERR_SCRATCH_LIMIT: return "batch needs more than the 16 MiB fixed scratch of mlra_decode_noalloc";
    case MLRA_ERR_DRAIN: return "in-flight device copies or MMAs did not finish after a failed wait: stop using this CUDA context";
    default: return "unknown status";
  }
}

int mlra_decode_profiled(mlra_handle h, const void* q, mlra_dtype q_dtype, const void* pool,
                         int num_pages, const int32_t* page_table, int pt_stride,
                         const int32_t* seq_lens, int batch, void* out, mlra_dtype out_dtype,
                         float* lse, void* workspace, size_t ws_bytes, void* const* events,
                         void* stream) {
  if (!out || !events) return MLRA_ERR_INVALID_ARG;
  for (int i = 0; i < 4; ++i)
    if (!events[i]) return MLRA_ERR_INVALID_ARG;
  return run_decode(h, q, q_dtype, pool, num_pages, page_table, pt_stride, seq_lens, batch, out, out_dtype,
                    lse, nullptr, workspace, ws_bytes, stream, 0, kWaitLimitNs, events);
}

// Test hook (not in the public header): a decode with one wait made to run out after
// `wait_limit_ns`, so the status word must report MLRA_ERR_TIMEOUT. where = 1: the decode
// kernel's producer withholds each CTA's first tile; where = 2: absorb CTA (1, 0) never issues
// its MMA (an error raised by a CTA other than the one that clears the status word). Used to
// check that a stalled pipeline ends with an error, not a hang, and that the error survives.
int mlra_test_decode_stalled(mlra_handle h, const void* q, mlra_dtype q_dtype, const void* pool,
                             int num_pages, const int32_t* page_table, int pt_stride,
                             const int32_t* seq_lens, int batch, void* out, void* workspace,
                             size_t ws_bytes, unsigned long long wait_limit_ns, int where, void* stream) {
  if (where != 1 && where != 2) return MLRA_ERR_INVALID_ARG;
  return run_decode(h, q, q_dtype, pool, num_pages, page_table, pt_stride, seq_lens, batch, out, MLRA_F32,
                    nullptr, nullptr, workspace, ws_bytes, stream, where, wait_limit_ns);
}

#ifdef MLRA_TRACE
// Profiling builds only: points the kernels' trace points at a device buffer of
// [3 kernels][1024 CTAs][512 points] uint64 (NULL turns tracing off).
int mlra_trace_set(void* device_buffer) {
  return cudaMemcpyToSymbol(g_mlra_trace, &device_buffer, sizeof(device_buffer)) == cudaSuccess
             ? MLRA_OK
             : MLRA_ERR_CUDA;
}
#endif

}  // extern "C"
