// producer.cuh - the step before the decode path: the cache row of each sequence's new token.
//
//   c   = x W^DKV              the token's latent, all k blocks ("Multi-Head Low-Rank
//                              Attention: Making Compressed Attention Actually Parallelizable",
//                              Core Mechanism: the input is projected into one latent per
//                              latent head; lesty.tech MLA article, section 4)
//   k^R = RoPE_pos(x W^KR)     its decoupled positional key, shared by every head (lesty.tech
//                              section 4), rotated as in RoFormer: pair (2i, 2i+1) by the angle
//                              pos * base^(-2i / d_r)
//   row [c | k^R] -> bf16 (or E4M3 bytes of v / scale for an E4M3 cache), slot pos % 64 of
//   page page_table[b][pos / 64]
//
// Both weight matrices are one bf16 matrix w_down [d_c + d_r][d_model], one row per output
// feature. Two kernels:
//   mlra_down_proj_kernel: split-K tcgen05 GEMM. One CTA per (128 output features, 128-wide
//     slice of d_model, batch tile): D^T[128 x NT] = W[128 x 128] X[NT x 128]^T, both operands
//     by TMA, K-major, accumulated in TMEM and written as fp32 partials [slice][b][feature].
//     Splitting d_model spreads the weight stream (the whole cost: it is read once) over all
//     SMs.
//   mlra_rope_append_kernel: four threads per (token, feature pair) sum the slices, one of them
//     rotates the RoPE pairs (angle in double precision: pos reaches 2^17), rounds to bf16 and
//     stores the pair into the token's page slot.
#pragma once

#include "common.cuh"

namespace mlra {

struct DownParams {
  int d_out;    // d_c + d_r
  int batch;
  float* part;  // [kslices][batch][d_out] fp32
  int* status;  // cleared by CTA (0, 0, 0); written by the append kernel
  EarlyTags tags;  // this kernel's errors (the append kernel folds them into status)
  unsigned long long wait_limit_ns;
};

template <int NT_>
struct DownShape {
  static constexpr int NT = NT_;
  static constexpr int KS = 128;                       // d_model slice per CTA
  static constexpr int NKR = 2;                        // 64-element swizzle regions per slice
  static constexpr int ROWB = 128;                     // bytes of a 64-element bf16 row
  static constexpr int A_REG = 128 * ROWB;             // 128 weight rows
  static constexpr int B_REG = NT * ROWB < 1024 ? 1024 : NT * ROWB;
  static constexpr int A_TX = NKR * 128 * ROWB;
  static constexpr int B_TX = NKR * NT * ROWB;
  static constexpr int OFF_BAR = NKR * A_REG + NKR * B_REG;
  static constexpr int SMEM = OFF_BAR + 64 + 1024;     // + alignment slack
  static constexpr int TMEM = NT <= 32 ? 32 : NT <= 64 ? 64 : 128;
  static constexpr int THREADS = 128;
  static_assert(NT % 16 == 0 && NT <= 128, "batch tile");
};

template <class Sh>
__global__ void __launch_bounds__(Sh::THREADS)
    mlra_down_proj_kernel(const __grid_constant__ CUtensorMap map_w, const __grid_constant__ CUtensorMap map_x,
                          const DownParams p) {
  constexpr int NT = Sh::NT;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* A = smem;
  uint8_t* B = smem + Sh::NKR * Sh::A_REG;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sh::OFF_BAR);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  const int mt = blockIdx.x, ks = blockIdx.y, n0 = blockIdx.z * NT;
  const int warp = warp_id(), lane = lane_id();
  bool mma_issued = false;  // (warp 0) the MMA went out: its commit is drained at teardown

  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
    // the weights do not depend on the previous kernel in the stream: load them first (rows
    // past d_out read as zero); the hidden states and the status word wait for it
    mbar_arrive_expect_tx(&bars[0], Sh::A_TX + Sh::B_TX);
    const uint64_t pol_w = l2_policy_evict_first();
    for (int r = 0; r < Sh::NKR; ++r)
      tma_load_2d(A + r * Sh::A_REG, &map_w, &bars[0], ks * Sh::KS + r * 64, mt * 128, pol_w);
    grid_dependency_wait();
    if (mt == 0 && ks == 0 && blockIdx.z == 0) clear_status_and_tags(p.status, p.tags);
    const uint64_t pol_x = l2_policy_evict_last();  // every 128-feature tile reads the same x
    for (int r = 0; r < Sh::NKR; ++r)
      tma_load_2d(B + r * Sh::B_REG, &map_x, &bars[0], ks * Sh::KS + r * 64, n0, pol_x);
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, Sh::TMEM);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dependency_wait();  // (returns at once: thread 0 has waited for the previous kernel)
  const uint32_t tbase = *tmem_slot;
  grid_launch_dependents();

  if (warp == 0) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[0], 0, abort_flag, p.wait_limit_ns));
    if (ok) {
      tc_fence_after();
      if (lane == 0) {
        constexpr uint32_t idesc = idesc_bf16_f32(128, NT, false, false);
#pragma unroll
        for (int k = 0; k < Sh::KS / 16; ++k) {
          const uint64_t a = smem_desc(smem_u32(A + (k / 4) * Sh::A_REG + (k % 4) * 32), 16, 8 * Sh::ROWB,
                                       swizzle_code(Sh::ROWB));
          const uint64_t b = smem_desc(smem_u32(B + (k / 4) * Sh::B_REG + (k % 4) * 32), 16, 8 * Sh::ROWB,
                                       swizzle_code(Sh::ROWB));
          umma_bf16(tbase, a, b, idesc, k > 0 ? 1u : 0u);
        }
        umma_commit(&bars[1]);
      }
      __syncwarp();
      mma_issued = true;
    }
  }
  const bool ok = mbar_wait(&bars[1], 0, abort_flag, p.wait_limit_ns);
  if (ok) {
    // D^T: TMEM lane = output feature (warp w reads lanes 32w..32w+31), column = batch row.
    // A warp's 32 lanes hold 32 consecutive features, so each store covers 128 contiguous bytes.
    tc_fence_after();
    const int f = mt * 128 + warp * 32 + lane;
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
#pragma unroll
    for (int c0 = 0; c0 < NT; c0 += 16) {
      float v[16];
      tmem_load_row<16>(tbase + lane_base + c0, v);
      tmem_ld_wait();
      if (f < p.d_out) {
#pragma unroll
        for (int n = 0; n < 16; ++n) {
          const int b = n0 + c0 + n;
          if (b < p.batch) p.part[((size_t)ks * p.batch + b) * p.d_out + f] = v[n];
        }
      }
    }
  }
  // drain before releasing TMEM and shared memory
  bool drained = true;
  if (threadIdx.x == 0) {
    drained = mbar_wait_drain(&bars[0], 0, p.wait_limit_ns);
    if (mma_issued) drained = mbar_wait_drain(&bars[1], 0, p.wait_limit_ns) && drained;
  }
  tc_fence_before();
  __syncthreads();
  // this kernel may fail before CTA (0, 0, 0) has cleared the status word: report by tag
  if (threadIdx.x == 0 && *abort_flag) report_early(p.tags, kTagTimeout);
  if (threadIdx.x == 0 && !drained) report_early(p.tags, kTagDrain);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, Sh::TMEM);
  }
}

struct AppendRowParams {
  const float* part;  // [kslices][batch][d_out]
  int kslices;
  int batch;
  int d_c, d_r, d_out;
  const int* positions;   // [batch]
  const int* page_table;  // [batch][pt_stride]
  int pt_stride;
  int num_pages;
  void* pool;             // [num_pages][64][d_out] bf16, or E4M3 bytes when fp8
  int fp8;                // E4M3 cache: store e4m3(v / scale)
  float latent_scale, rope_scale;
  double log2_base;       // log2 of the RoPE base
  int* status;
  EarlyTags tags;         // the down-projection kernel's errors, folded in by block 0
};

// Block (kAppendPairs, kAppendGroups): x = feature pair of one token, y = one of the groups of
// d_model slices that are summed separately (slices y, y + groups, ...), then combined through
// shared memory. Loads of one slice by a warp cover 256 contiguous bytes.
constexpr int kAppendPairs = 64;
constexpr int kAppendGroups = 4;

__global__ void __launch_bounds__(kAppendPairs * kAppendGroups) mlra_rope_append_kernel(const AppendRowParams p) {
  __shared__ float2 red[kAppendGroups][kAppendPairs];
  grid_dependency_wait();  // the partials come from the down-projection kernel
  if (blockIdx.x == 0 && threadIdx.x == 0 && threadIdx.y == 0) fold_early(p.tags, p.status);
  const int pairs = p.d_out / 2;
  const int idx = blockIdx.x * kAppendPairs + threadIdx.x;
  const bool live = idx < p.batch * pairs;
  const int b = live ? idx / pairs : 0;
  const int f0 = live ? 2 * (idx % pairs) : 0;
  // the slot's page id is read from a clamped index (always inside the row) so that its load
  // overlaps the partial sums below; the checks come before the store
  const int pos = live ? __ldg(p.positions + b) : 0;
  const int cap = p.pt_stride * kPage;
  const int page = live ? __ldg(p.page_table + (size_t)b * p.pt_stride + min(max(pos, 0), cap - 1) / kPage) : 0;
  constexpr int U = 4;  // independent loads in flight per thread
  const size_t slice = (size_t)p.batch * p.d_out;
  const float* src = p.part + (size_t)b * p.d_out + f0;
  float a0[U], a1[U];
#pragma unroll
  for (int u = 0; u < U; ++u) a0[u] = a1[u] = 0.f;
  if (live) {
    int s = threadIdx.y;
    for (; s + (U - 1) * kAppendGroups < p.kslices; s += U * kAppendGroups) {
      float2 t[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        t[u] = __ldcg(reinterpret_cast<const float2*>(src + (size_t)(s + u * kAppendGroups) * slice));
#pragma unroll
      for (int u = 0; u < U; ++u) {
        a0[u] += t[u].x;
        a1[u] += t[u].y;
      }
    }
    for (; s < p.kslices; s += kAppendGroups) {
      const float2 t = __ldcg(reinterpret_cast<const float2*>(src + (size_t)s * slice));
      a0[0] += t.x;
      a1[0] += t.y;
    }
  }
  float2 part = make_float2(0.f, 0.f);
#pragma unroll
  for (int u = 0; u < U; ++u) {
    part.x += a0[u];
    part.y += a1[u];
  }
  red[threadIdx.y][threadIdx.x] = part;
  __syncthreads();
  if (threadIdx.y != 0 || !live) return;
  float v0 = 0.f, v1 = 0.f;
#pragma unroll
  for (int g = 0; g < kAppendGroups; ++g) {
    v0 += red[g][threadIdx.x].x;
    v1 += red[g][threadIdx.x].y;
  }
  if (pos < 0 || pos >= cap) {
    set_status(p.status, kErrSeqLen);
    return;
  }
  if (page < 0 || page >= p.num_pages) {
    set_status(p.status, kErrPageOob);
    return;
  }
  if (f0 >= p.d_c) {
    const int i = (f0 - p.d_c) / 2;
    const double ang = (double)pos * exp2(-2.0 * i / p.d_r * p.log2_base);
    double sn, cs;
    sincos(ang, &sn, &cs);
    const float cf = (float)cs, sf = (float)sn;
    const float r0 = v0 * cf - v1 * sf;
    const float r1 = v0 * sf + v1 * cf;
    v0 = r0;
    v1 = r1;
  }
  const size_t at = ((size_t)page * kPage + pos % kPage) * p.d_out + f0;
  if (p.fp8) {
    const float sc = f0 < p.d_c ? p.latent_scale : p.rope_scale;
    *reinterpret_cast<uint16_t*>(static_cast<uint8_t*>(p.pool) + at) = e4m3x2_from_f32(__fdiv_rn(v0, sc), __fdiv_rn(v1, sc));
  } else {
    *reinterpret_cast<uint32_t*>(static_cast<__nv_bfloat16*>(p.pool) + at) = pack_bf16x2(v0, v1);
  }
}

}  // namespace mlra
