// decode.cuh - split-KV latent attention for one decode step (the hot loop).
//
// One CTA serves one (group g, latent block j, head chunk) triple. A group owns a run of
// 128-token tiles of the flattened (sequence, tile) list (see the planner in common.cuh);
// the CTAs of a group run side by side over the same tiles, each on its own latent block,
// so the shared RoPE key rows they all read are served from L2 after the first read.
//
// Per 128-token tile, with the query absorbed into the block's latent space
// (lesty.tech MLA article, section 5, "On-The-Fly Matrix Absorption"):
//   S^T[t][h] = [c_j | k^R][t] . [q~_h | q^R_h]      tcgen05 MMA, M = 128 tokens, N = heads,
//                                                    K = d_b + d_r, fp32 accumulator in TMEM
//   online softmax over t (base 2; q was pre-scaled by scale * log2 e)
//   O^T[f][h] += sum_t c_j[t][f] P^T[t][h]           tcgen05 MMA, M = 128 latent features,
//                                                    N = heads, K = 128 tokens
// Tokens sit on the MMA's M dimension because a block serves only h/k heads (32 for MLRA-4),
// fewer than the 64/128 rows an MMA needs.
//
// Roles (96 + 128*NWG threads): warp 0 issues TMA loads of pages and queries, warp 1
// allocates TMEM and issues the QK MMAs, warps 2 .. 1+4*NWG form NWG softmax warpgroups (each
// owns a slice of the heads) that run the softmax and write the partial results, and the last
// warp issues the PV MMAs. Each issuer tracks its own MMAs with its own tcgen05.commit
// barriers. The roles hand off through mbarriers; each wait is bounded (see mbar_wait).
//
// Softmax detail: each thread owns one token row of S^T and all its heads. The running
// maximum m_h is only raised when some score exceeds it by more than the shape's SLACK (in
// log2 units); otherwise P = exp2(s - m_h) is used as is (values up to 2^slack stay inside
// the range of P's storage type). A raise costs a cross-thread max and a rescale of O in TMEM; it happens
// on a segment's first tile and then rarely.
#pragma once

#include "common.cuh"

namespace mlra {


__host__ __device__ constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }

template <int DB_, int DR_, int NP_, int STAGES_, int QBUF_, int PBUF_, int SBUF_ = 2, bool FP8_ = false,
          int NWG_ = 2, int TPS_ = 1>
struct DecodeShape {
  static constexpr int DB = DB_;      // latent block width d_c / k
  static constexpr int DR = DR_;      // RoPE key width
  static constexpr int NP = NP_;      // heads per CTA, 16 / 32 / 64
  // E4M3 cache: every cached element is one byte, and the MMAs run on E4M3 operands. The query
  // and P are then each carried as two E4M3 terms (hi + lo) in two column sets of N, so N = 2 NP
  // (an MMA costs the same up to N = 128).
  static constexpr bool FP8 = FP8_;
  static constexpr int EB = FP8 ? 1 : 2;   // bytes per cached element
  static constexpr int NQ = FP8 ? 2 : 1;   // query / P terms per head
  static constexpr int MN = NQ * NP;       // MMA N
  static constexpr int KT = 32 / EB;       // tokens per PV K step (32 bytes of K per MMA)
  // P is written as p * P_SCALE (E4M3 split), with the lazy maximum's slack lowered so that
  // p * P_SCALE <= 2^(SLACK + log2 P_SCALE) = 256 stays inside E4M3's range
  static constexpr float SLACK = FP8 ? 3.0f : 8.0f;
  static constexpr float P_SCALE = FP8 ? 32.0f : 1.0f;
  static constexpr int NWG = NWG_;    // softmax warpgroups; each owns NP / NWG heads
  static constexpr int HW = NP / NWG;
  static constexpr int PV_WARP = 2 + 4 * NWG;  // after the softmax warps
  // named barriers: 1 + 2g and 2 + 2g for softmax warpgroup g, then the segment-list hand-off
  static constexpr int PLAN_BAR = 2 * NWG + 1;
  static constexpr int THREADS = 32 * (PV_WARP + 1);
  static constexpr int STAGES = STAGES_;
  // Tiles per pipeline stage: a stage is TPS consecutive tile slots loaded and freed through
  // one barrier phase (a phase per 128-token tile costs more than the copies of a small tile
  // need). Slot i of the ring holds tile i's pages; the last tile of a launch may leave a
  // stage part-filled.
  static constexpr int TPS = TPS_;
  static constexpr int SLOTS = STAGES * TPS;
  static constexpr int QBUF = QBUF_;  // query buffers
  // probability buffers; 0: P(i) is written over the RoPE columns of tile i's own stage,
  // which QK(i) has finished reading when the softmax sees S(i), and the stage is only
  // reloaded after PV(i) has read it
  static constexpr int PBUF = PBUF_;
  static constexpr bool P_IN_STAGE = PBUF == 0;
  // Depth of the P-ready / PV-done barrier rings. Tile i's softmax can only run once PV(i -
  // STAGES) has freed tile i's stage, so with at least STAGES slots no ring slot is armed again
  // before the phase it held has been waited for (no parity aliasing), however far the softmax
  // runs ahead of the PV issuer.
  static constexpr int PR = SLOTS > 2 ? SLOTS : 2;
  // A cache row is split into swizzle-width regions (at most 128 bytes): block columns and RoPE
  // columns.
  static constexpr int CW = DB * EB < 128 ? DB : 128 / EB;
  static constexpr int NC = DB / CW;
  static constexpr int RW = DR * EB < 128 ? DR : 128 / EB;
  static constexpr int NR = DR / RW;
  static constexpr int C_ROWB = CW * EB;
  static constexpr int R_ROWB = RW * EB;
  static constexpr int C_REG = round_up(kTile * C_ROWB, 1024);
  static constexpr int R_REG = round_up(kTile * R_ROWB, 1024);
  static constexpr int STAGE_BYTES = NC * C_REG + NR * R_REG;
  static constexpr int PAGE_TX = NC * kPage * C_ROWB + NR * kPage * R_ROWB;
  static constexpr int QC_REG = round_up(MN * C_ROWB, 1024);
  static constexpr int QR_REG = round_up(MN * R_ROWB, 1024);
  static constexpr int Q_BYTES = NC * QC_REG + NR * QR_REG;
  static constexpr int P_ROWB = NP * 2;  // NP bf16, or NQ * NP E4M3 bytes
  static constexpr int P_BYTES = round_up(kTile * P_ROWB, 1024);
  static constexpr int NMT = DB >= 128 ? DB / 128 : 1;  // PV M tiles
  // A stage is loaded and freed in NG groups, one per PV M tile (128 latent features); the RoPE
  // columns, and P written over them, belong to the last group. A group is reloaded as soon as
  // the PV MMAs of its M tile have read it, so with several M tiles (d_b = 256, 512) the next
  // tile's first columns stream in while this tile's PV is still running.
  static constexpr int NG = NMT;
  static constexpr int RPG = NC / NMT;  // block regions per group
  static constexpr uint32_t PV_LBO = DB >= 128 ? C_REG : 0;  // next 64-feature chunk
  static constexpr int SBUF = SBUF_;                // S buffers of MN columns in TMEM
  static constexpr int S_COL0 = 0;
  static constexpr int O_COL = SBUF * MN;           // NMT x MN columns
  static constexpr int TMEM_USED = SBUF * MN + NMT * MN;
  static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 :
                                   TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static constexpr int MAX_SEGS = 64;
  // small shared state after the big buffers
  static constexpr int OFF_STAGES = 0;
  static constexpr int OFF_Q = OFF_STAGES + SLOTS * STAGE_BYTES;
  static constexpr int OFF_P = OFF_Q + QBUF * Q_BYTES;
  // The running max per head is the same in every softmax thread. With 32 heads per warpgroup
  // each warp keeps one copy in shared memory (read as broadcasts, written only when raised),
  // which saves 32 registers per thread; with fewer heads it stays in registers.
  static constexpr bool M_SMEM = HW >= 32;
  static constexpr int OFF_M = OFF_P + PBUF * P_BYTES;          // running max: HW floats per softmax warp
  static constexpr int OFF_RED = OFF_M + 4 * NWG * HW * 4;      // 4 x NP floats
  static constexpr int OFF_SEG = OFF_RED + 4 * NP * 4;          // MAX_SEGS segments
  static constexpr int OFF_BAR = round_up(OFF_SEG + MAX_SEGS * 16, 8);
  static constexpr int NUM_BARS = 2 * STAGES * NG + 2 * QBUF + 2 * SBUF + 2 * PR + 2;
  // bytes one page brings into group g
  static constexpr int group_tx(int g) { return RPG * kPage * C_ROWB + (g == NG - 1 ? NR * kPage * R_ROWB : 0); }
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;       // tmem slot, flags, scratch
  static constexpr int SMEM_BYTES = OFF_MISC + 64 * 4 + 1024;  // + alignment slack
  static_assert(DB % CW == 0 && DR % RW == 0, "region split");
  static_assert(NP == 16 || NP == 32 || NP == 64, "heads per CTA");
  static_assert(NWG >= 1 && NWG <= 7 && NP % NWG == 0 && HW % 8 == 0, "softmax warpgroups");
  static_assert(!FP8 || (NMT == 1 && MN <= 128 && R_ROWB == 64), "E4M3 shapes: one PV M tile, 64-byte RoPE rows");
  static_assert(QBUF == 1 || QBUF == 2, "query buffers");
  static_assert(SBUF >= 2 && TMEM_USED <= 512, "S buffers");
  static_assert(SMEM_BYTES <= 227 * 1024, "dynamic shared memory of one sm_100 CTA");
  static_assert(NG * RPG == NC && STAGES * NG <= 32, "column groups");
  static_assert(PBUF == 0 || PBUF == 1 || PBUF == 2, "P buffers");
  static_assert(PBUF != 0 || P_BYTES <= NR * R_REG, "P must fit the RoPE region of a stage");
};

struct DecodeParams {
  const int* seq_lens;
  const int* page_table;
  int pt_stride;
  int batch;
  int num_pages;
  int groups;       // CTA groups
  int nsub;         // CTAs per group = k * chunks
  int chunks;       // head chunks per block
  int heads_block;  // h / k
  int h;            // total heads
  int d_c;          // column of k^R in a cache row
  int q_rows;       // query rows a CTA loads: min(h/k, NP); rows past them stay zero
  const float* qfac;  // E4M3 cache: [batch][nsub][NP] factor of each head's query terms
  float o_scale;    // E4M3 cache: latent scale / P scale, applied to the partial outputs
  float* o_part;    // [slots][h][DB] fp32, normalised partial latent outputs
  float* lse_part;  // [slots][h] fp32, log2-domain log-sum-exp
  int* status;
  EarlyTags tags;    // errors of the absorb kernel (folded in by CTA 0)
  unsigned long long wait_limit_ns;
  int inject_stall;  // test hook: 1 = the producer withholds its first tile
};

// Reduce N per-head values across the 32 lanes of a warp and scatter the results: afterwards
// lane l holds in v[0..max(1, N/32)) the reduction over all lanes of heads
// [l*N/32, (l+1)*N/32) when N >= 32, or of head (l mod N) when N < 32.
template <bool IS_MAX>
__device__ __forceinline__ float red_op(float a, float b) {
  return IS_MAX ? fmaxf(a, b) : a + b;
}
template <int OFF, int N, bool IS_MAX, int L>
__device__ __forceinline__ void rs_step(float (&v)[L], int lane) {
  const bool upper = (lane & OFF) != 0;
#pragma unroll
  for (int x = 0; x < N / 2; ++x) {
    const float send = upper ? v[x] : v[x + N / 2];
    const float keep = upper ? v[x + N / 2] : v[x];
    v[x] = red_op<IS_MAX>(keep, __shfl_xor_sync(0xffffffffu, send, OFF));
  }
}
template <int OFF, int N, bool IS_MAX, int L>
__device__ __forceinline__ void rs_chain(float (&v)[L], int lane) {
  if constexpr (OFF >= 1 && N >= 2) {
    rs_step<OFF, N, IS_MAX>(v, lane);
    rs_chain<OFF / 2, N / 2, IS_MAX>(v, lane);
  }
}
template <int OFF, int N, bool IS_MAX, int L>
__device__ __forceinline__ void plain_chain(float (&v)[L]) {
  if constexpr (OFF >= N) {
#pragma unroll
    for (int x = 0; x < N; ++x) v[x] = red_op<IS_MAX>(v[x], __shfl_xor_sync(0xffffffffu, v[x], OFF));
    plain_chain<OFF / 2, N, IS_MAX>(v);
  }
}
template <int N, bool IS_MAX>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[N], int lane) {
  if constexpr (N >= 32) {
    rs_chain<16, N, IS_MAX>(v, lane);
  } else {
    plain_chain<16, N, IS_MAX>(v);  // fold lanes that differ above bit log2(N)
    rs_chain<N / 2, N, IS_MAX>(v, lane);
  }
}
// Writes the scattered per-head values of this lane to dst[h].
template <int N>
__device__ __forceinline__ void store_scattered(const float (&v)[N], float* dst, int lane) {
  if constexpr (N < 32) {
    if (lane < N) dst[lane] = v[0];
  } else {
#pragma unroll
    for (int x = 0; x < N / 32; ++x) dst[lane * (N / 32) + x] = v[x];
  }
}

// Pairwise fp32 ops on the packed f32x2 datapath.
__device__ __forceinline__ unsigned long long f2pack(float a, float b) {
  return (static_cast<unsigned long long>(__float_as_uint(b)) << 32) | __float_as_uint(a);
}
__device__ __forceinline__ void sub_f32x2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2pack(a0, a1)), "l"(f2pack(b0, b1)));
  d0 = __uint_as_float(static_cast<uint32_t>(d));
  d1 = __uint_as_float(static_cast<uint32_t>(d >> 32));
}
__device__ __forceinline__ void add_f32x2(float& d0, float& d1, float a0, float a1, float b0, float b1) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2pack(a0, a1)), "l"(f2pack(b0, b1)));
  d0 = __uint_as_float(static_cast<uint32_t>(d));
  d1 = __uint_as_float(static_cast<uint32_t>(d >> 32));
}

// One MMA of the shape's kind: bf16 (K = 16) or E4M3 (K = 32).
template <class Sh>
__device__ __forceinline__ void shape_mma(uint32_t d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  if constexpr (Sh::FP8)
    umma_e4m3(d, a, b, idesc, acc);
  else
    umma_bf16(d, a, b, idesc, acc);
}

// Ring position of tile i: its slot (shared-memory tile), its stage (barriers) and the parity
// of the stage's phase that carries it.
template <class Sh>
__device__ __forceinline__ uint32_t tile_slot(uint32_t i) {
  return ((i / Sh::TPS) % Sh::STAGES) * Sh::TPS + i % Sh::TPS;
}
template <class Sh>
__device__ __forceinline__ uint32_t tile_stage(uint32_t i) {
  return (i / Sh::TPS) % Sh::STAGES;
}
template <class Sh>
__device__ __forceinline__ uint32_t tile_phase(uint32_t i) {
  return ((i / Sh::TPS) / Sh::STAGES) & 1;
}

template <class Sh>
__global__ void __launch_bounds__(Sh::THREADS, 1)
    mlra_decode_kernel(const __grid_constant__ CUtensorMap map_c,
                       const __grid_constant__ CUtensorMap map_r,
                       const __grid_constant__ CUtensorMap map_qc,
                       const __grid_constant__ CUtensorMap map_qr, const DecodeParams p) {
  constexpr int NP = Sh::NP, STAGES = Sh::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  MLRA_TRACE_INIT
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stages = smem + Sh::OFF_STAGES;
  uint8_t* qbufs = smem + Sh::OFF_Q;
  uint8_t* pbufs = smem + Sh::OFF_P;
  float* red_sm = reinterpret_cast<float*>(smem + Sh::OFF_RED);
  Segment* segs = reinterpret_cast<Segment*>(smem + Sh::OFF_SEG);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sh::OFF_BAR);
  uint64_t* full_bar = bars;                         // [stage][group]
  uint64_t* empty_bar = bars + STAGES * Sh::NG;       // [stage][group]
  uint64_t* qfull_bar = bars + 2 * STAGES * Sh::NG;
  uint64_t* qempty_bar = qfull_bar + Sh::QBUF;
  uint64_t* sfull_bar = qempty_bar + Sh::QBUF;
  uint64_t* sfree_bar = sfull_bar + Sh::SBUF;
  uint64_t* pfull_bar = sfree_bar + Sh::SBUF;
  uint64_t* pvdone_bar = pfull_bar + Sh::PR;
  uint64_t* mmadone_bar = pvdone_bar + Sh::PR;  // [0] QK issuer, [1] PV issuer
  int* misc = reinterpret_cast<int*>(smem + Sh::OFF_MISC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = misc + 1;
  int* plan_err = misc + 2;
  int* scratch = misc + 8;  // 40 ints for the planner
  volatile int* plan_words = misc + 48;  // segment count and resume point of the first list
  volatile int* drain_err = misc + 3;     // a teardown drain ran out of time

  const int warp = warp_id(), lane = lane_id();
  const int group = blockIdx.x / p.nsub;
  const int sub = blockIdx.x % p.nsub;
  const int blk = sub / p.chunks;
  const int chunk = sub % p.chunks;
  const int head0 = blk * p.heads_block + chunk * NP;
  const int nheads = min(NP, p.heads_block - chunk * NP);
  const int cap_len = p.pt_stride * kPage;
  if (threadIdx.x == 0) MLRA_TRACE_POINT(1, 0);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES * Sh::NG; ++s) {
      mbar_init(&full_bar[s], Sh::TPS);  // one arrival per tile of the stage
      mbar_init(&empty_bar[s], 1);
    }
    for (int s = 0; s < Sh::QBUF; ++s) {
      mbar_init(&qfull_bar[s], 1);
      mbar_init(&qempty_bar[s], 1);
    }
    for (int s = 0; s < Sh::SBUF; ++s) {
      mbar_init(&sfull_bar[s], 1);
      mbar_init(&sfree_bar[s], 4 * Sh::NWG);
    }
    for (int s = 0; s < Sh::PR; ++s) {
      mbar_init(&pfull_bar[s], 4 * Sh::NWG);
      mbar_init(&pvdone_bar[s], 1);
    }
    mbar_init(&mmadone_bar[0], 1);
    mbar_init(&mmadone_bar[1], 1);
    *abort_flag = 0;
    *plan_err = 0;
    *drain_err = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&map_c);
    tma_prefetch_map(&map_r);
    tma_prefetch_map(&map_qc);
    tma_prefetch_map(&map_qr);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Sh::TMEM_COLS);
    tmem_relinquish();
  }
  if (p.q_rows < NP) {
    // Head chunks narrower than the MMA's N (h/k < NP): the query loads bring q_rows rows, and
    // the rows past them, which no load ever writes, are zero for the whole launch. A swizzled
    // row keeps its bytes within its own row span, so whole rows are cleared.
    for (int qb = 0; qb < Sh::QBUF; ++qb) {
      uint8_t* qdst = qbufs + qb * Sh::Q_BYTES;
      for (int r = 0; r < Sh::NC; ++r)
        for (int i = p.q_rows * Sh::C_ROWB + threadIdx.x * 16; i < NP * Sh::C_ROWB; i += Sh::THREADS * 16)
          *reinterpret_cast<uint4*>(qdst + r * Sh::QC_REG + i) = make_uint4(0, 0, 0, 0);
      for (int r = 0; r < Sh::NR; ++r)
        for (int i = p.q_rows * Sh::R_ROWB + threadIdx.x * 16; i < NP * Sh::R_ROWB; i += Sh::THREADS * 16)
          *reinterpret_cast<uint4*>(qdst + Sh::NC * Sh::QC_REG + r * Sh::QR_REG + i) = make_uint4(0, 0, 0, 0);
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;
  if (threadIdx.x == 0) MLRA_TRACE_POINT(1, 1);
  // the combine kernel may be scheduled as soon as SMs free up; it waits for this grid's
  // partials before reading them
  grid_launch_dependents();

  // ---- plan: which flattened tiles this group owns (seq_lens do not depend on the
  // previous kernel, so this overlaps its tail under programmatic dependent launch) ----
  // Batches up to 32 * kPlanPer: every warp scans seq_lens on its own (no block barrier) and
  // warp 0 writes the segment list; larger batches use block-wide scans.
  int err = 0;
  WarpPlan wp;
  const bool warp_plan = warp_plan_load(p.seq_lens, p.batch, cap_len, wp, &err);
  const int T = warp_plan ? wp.total : block_total_tiles(p.seq_lens, p.batch, cap_len, scratch, &err);
  const int quota = T > 0 ? (T + p.groups - 1) / p.groups : 1;
  const int lo = min(group * quota, T);
  const int hi = min(lo + quota, T);
  if (err) atomicOr(plan_err, 1);

  // pipeline counters persist across segment-list refills
  uint32_t it = 0;      // tiles consumed/produced so far by this role
  uint32_t segc = 0;    // segments so far
  // producer: which (stage, group) barriers have a load issued and the parity of the last
  // issued phase of each, for the drain at the end
  uint32_t issued_mask = 0, issued_phase = 0;
  // softmax-role partial sums (the warpgroup's heads)
  float l_part[Sh::HW];
#pragma unroll
  for (int x = 0; x < Sh::HW; ++x) l_part[x] = 0.f;

  // first segment list from the warp plan: warp 0 builds it and hands it over through a
  // named barrier, so it goes on to issue loads while the other warps pick the list up
  int first_total = 0, first_rb = p.batch, first_rp = 0;
  if (warp_plan && lo < hi) {
    if (warp == 0) {
      first_total = warp_plan_segments(wp, lo, hi, segs, Sh::MAX_SEGS, &first_rb, &first_rp);
      if (lane == 0) {
        plan_words[0] = first_total;
        plan_words[1] = first_rb;
        plan_words[2] = first_rp;
      }
      __threadfence_block();
      __syncwarp();
      named_bar_arrive(Sh::PLAN_BAR, Sh::THREADS);
    } else {
      named_bar_sync(Sh::PLAN_BAR, Sh::THREADS);
      first_total = plan_words[0];
      first_rb = plan_words[1];
      first_rp = plan_words[2];
    }
  }

  int b_start = 0, p_start = 0;
  bool more = lo < hi;
  bool first_list = true;
  while (more) {
    int nseg, rb = p.batch, rp = 0;
    if (first_list && warp_plan) {
      nseg = min(first_total, Sh::MAX_SEGS);
      more = first_total > Sh::MAX_SEGS;
      rb = first_rb;
      rp = first_rp;
    } else {
      int more_i;
      nseg = block_collect_segments(p.seq_lens, p.batch, cap_len, lo, hi, b_start, p_start, segs,
                                    Sh::MAX_SEGS, scratch, &more_i, &rb, &rp, &err);
      more = more_i != 0;
    }
    first_list = false;
    b_start = rb;
    p_start = rp;
    if (threadIdx.x == 0) MLRA_TRACE_POINT(1, 2);

    if (warp == 0) {
      // ============================== TMA producer ==============================
      const uint64_t pol_stream = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      grid_dependency_wait();  // q_pack and the reset status word come from the absorb kernel
      if (lane == 0) MLRA_TRACE_POINT(1, 3);
      if (lane == 0 && *plan_err) set_status(p.status, kErrSeqLen);
      for (int si = 0; si < nseg && !*abort_flag; ++si) {
        const Segment sg = segs[si];
        const int pages_b = (sg.n + kPage - 1) / kPage;
        bool ok = true;
        if (lane == 0) {
          const int qb = segc % Sh::QBUF;
          ok = mbar_wait(&qempty_bar[qb], ((segc / Sh::QBUF) & 1) ^ 1, abort_flag, p.wait_limit_ns);
          if (ok) {
            uint8_t* qdst = qbufs + qb * Sh::Q_BYTES;
            mbar_arrive_expect_tx(&qfull_bar[qb], Sh::NQ * p.q_rows * (Sh::DB + Sh::DR) * Sh::EB);
            const int qrow = (sg.b * p.nsub + sub) * Sh::MN;
            for (int r = 0; r < Sh::NC; ++r)
              tma_load_2d(qdst + r * Sh::QC_REG, &map_qc, &qfull_bar[qb], r * Sh::CW, qrow, pol_keep);
            for (int r = 0; r < Sh::NR; ++r)
              tma_load_2d(qdst + Sh::NC * Sh::QC_REG + r * Sh::QR_REG, &map_qr, &qfull_bar[qb],
                          Sh::DB + r * Sh::RW, qrow, pol_keep);
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        ++segc;
        // Page ids of this segment, a 64-page window held two registers per lane; the loads
        // for the upper half are issued 16 tiles before they are needed, so the producer
        // never waits on a page-table read.
        const int* pt_row = p.page_table + (size_t)sg.b * p.pt_stride;
        int wb = 2 * sg.tile_begin;
        auto load_ids = [&](int base) {
          const int pp = base + lane;
          return pp < pages_b ? __ldg(pt_row + pp) : 0;
        };
        int w0 = load_ids(wb), w1 = load_ids(wb + 32);
        auto page_id = [&](int pg) {  // warp-uniform pg in [wb, wb + 64); only the half
                                       // that holds pg is read, so a fresh load of the other
                                       // half is not waited for
          if (pg - wb < 32) return __shfl_sync(0xffffffffu, w0, pg - wb);
          return __shfl_sync(0xffffffffu, w1, pg - wb - 32);
        };
        for (int t = sg.tile_begin; t < sg.tile_end; ++t, ++it) {
          const int p0 = 2 * t;
          if (p0 >= wb + 32) {  // slide the window by 32 pages
            wb += 32;
            w0 = w1;
            w1 = load_ids(wb + 32);
          }
          int id0 = page_id(p0);
          const int npg = (p0 + 1 < pages_b) ? 2 : 1;
          int id1 = page_id(min(p0 + 1, pages_b - 1));
          ok = true;
          if (lane == 0) {
            if (id0 < 0 || id0 >= p.num_pages) { set_status(p.status, kErrPageOob); id0 = 0; }
            if (npg == 2 && (id1 < 0 || id1 >= p.num_pages)) { set_status(p.status, kErrPageOob); id1 = 0; }
            const int st = tile_stage<Sh>(it);
            const uint32_t ph = tile_phase<Sh>(it);
            uint8_t* dst = stages + tile_slot<Sh>(it) * Sh::STAGE_BYTES;
            for (int g = 0; g < Sh::NG && ok; ++g) {
              const int gi = st * Sh::NG + g;
              // the stage's previous phase must be freed before its first tile is loaded
              if (it % Sh::TPS == 0) ok = mbar_wait(&empty_bar[gi], ph ^ 1, abort_flag, p.wait_limit_ns);
              if (ok && !(p.inject_stall == 1 && it == 0)) {
                if (g == 0) MLRA_TRACE_POINT(1, 8 + min((int)it, 31));
                mbar_arrive_expect_tx(&full_bar[gi], npg * Sh::group_tx(g));
                issued_mask |= 1u << gi;
                issued_phase = (issued_phase & ~(1u << gi)) | (ph << gi);
                for (int pg = 0; pg < npg; ++pg) {
                  const int y = (pg ? id1 : id0) * kPage;
                  for (int r = g * Sh::RPG; r < (g + 1) * Sh::RPG; ++r)
                    tma_load_2d(dst + r * Sh::C_REG + pg * kPage * Sh::C_ROWB, &map_c, &full_bar[gi],
                                blk * Sh::DB + r * Sh::CW, y, pol_stream);
                  if (g == Sh::NG - 1)
                    for (int r = 0; r < Sh::NR; ++r)
                      tma_load_2d(dst + Sh::NC * Sh::C_REG + r * Sh::R_REG + pg * kPage * Sh::R_ROWB,
                                  &map_r, &full_bar[gi], p.d_c + r * Sh::RW, y, pol_keep);
                }
              }
            }
          }
          if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        }
      }
      // A launch whose last tile leaves its stage part-filled completes that stage's phase with
      // count-only arrivals (the QK issuer waits for it; the teardown drains it).
      if (Sh::TPS > 1 && lane == 0 && it % Sh::TPS != 0 && (!more || *abort_flag)) {
        const int st = tile_stage<Sh>(it - 1);
        for (int g = 0; g < Sh::NG; ++g)
          for (uint32_t x = it % Sh::TPS; x < (uint32_t)Sh::TPS; ++x) mbar_arrive(&full_bar[st * Sh::NG + g]);
      }
    } else if (warp == 1) {
      // ============================== QK issuer ==============================
      // One thread issues S^T(i) = [c_j | k^R](i) [q~ | q^R]^T once tile i's pages (and, at a
      // segment start, its query) have landed and the softmax has read the S buffer's previous
      // contents. The PVs have their own issuing warp, so a finished P never waits behind a
      // QK wait here.
      if (lane == 0) {
        constexpr uint32_t idesc_qk = Sh::FP8 ? idesc_e4m3_f32(128, Sh::MN, false, false)
                                              : idesc_bf16_f32(128, NP, false, false);
        uint32_t ci = it, sc = segc;
        bool ok = true;
        for (int si = 0; si < nseg && ok; ++si) {
          const Segment sg = segs[si];
          const int qb = sc % Sh::QBUF;
          ok = mbar_wait(&qfull_bar[qb], (sc / Sh::QBUF) & 1, abort_flag, p.wait_limit_ns);
          for (int t = sg.tile_begin; t < sg.tile_end && ok; ++t, ++ci) {
            if (ci >= Sh::SBUF)
              ok = mbar_wait(&sfree_bar[ci % Sh::SBUF], ((ci / Sh::SBUF) - 1) & 1, abort_flag, p.wait_limit_ns);
            MLRA_TRACE_POINT(1, 432 + min((int)ci, 31));
            const uint32_t st_addr = smem_u32(stages + tile_slot<Sh>(ci) * Sh::STAGE_BYTES);
            const uint32_t q_addr = smem_u32(qbufs + qb * Sh::Q_BYTES);
            const uint32_t d = tbase + Sh::S_COL0 + (ci % Sh::SBUF) * Sh::MN;
            uint32_t acc = 0;
            // each column group's MMAs go out as soon as that group has landed
#pragma unroll
            for (int g = 0; g < Sh::NG; ++g) {
              if (ok) ok = mbar_wait(&full_bar[tile_stage<Sh>(ci) * Sh::NG + g], tile_phase<Sh>(ci), abort_flag, p.wait_limit_ns);
              if (!ok) break;
              if (g == 0) MLRA_TRACE_POINT(1, 400 + min((int)ci, 31));
              tc_fence_after();
#pragma unroll
              for (int r = g * Sh::RPG; r < (g + 1) * Sh::RPG; ++r) {
#pragma unroll
                for (int ks = 0; ks < Sh::C_ROWB / 32; ++ks) {
                  const uint64_t a = smem_desc(st_addr + r * Sh::C_REG + ks * 32, 16, 8 * Sh::C_ROWB,
                                               swizzle_code(Sh::C_ROWB));
                  const uint64_t b = smem_desc(q_addr + r * Sh::QC_REG + ks * 32, 16, 8 * Sh::C_ROWB,
                                               swizzle_code(Sh::C_ROWB));
                  shape_mma<Sh>(d, a, b, idesc_qk, acc);
                  acc = 1;
                }
              }
              if (g == Sh::NG - 1) {
#pragma unroll
                for (int r = 0; r < Sh::NR; ++r) {
#pragma unroll
                  for (int ks = 0; ks < Sh::R_ROWB / 32; ++ks) {
                    const uint64_t a = smem_desc(st_addr + Sh::NC * Sh::C_REG + r * Sh::R_REG + ks * 32, 16,
                                                 8 * Sh::R_ROWB, swizzle_code(Sh::R_ROWB));
                    const uint64_t b = smem_desc(q_addr + Sh::NC * Sh::QC_REG + r * Sh::QR_REG + ks * 32, 16,
                                                 8 * Sh::R_ROWB, swizzle_code(Sh::R_ROWB));
                    shape_mma<Sh>(d, a, b, idesc_qk, 1);
                  }
                }
              }
            }
            MLRA_TRACE_POINT(1, 40 + min((int)ci, 31));
            if (!ok) break;
            umma_commit(&sfull_bar[ci % Sh::SBUF]);
            if (t == sg.tile_end - 1) umma_commit(&qempty_bar[qb]);
          }
          ++sc;
        }
        segc = sc;
      }
      __syncwarp();
      uint32_t list_tiles = 0;
      for (int i = 0; i < nseg; ++i) list_tiles += segs[i].tile_end - segs[i].tile_begin;
      it += list_tiles;
      segc = __shfl_sync(0xffffffffu, segc, 0);
    } else if (warp == Sh::PV_WARP) {
      // ============================== PV issuer ==============================
      // One thread issues O^T += C_j^T(i) P^T(i) as soon as both softmax warpgroups have
      // written P(i), then frees tile i's pipeline stage and signals pvdone.
      if (lane == 0) {
        constexpr uint32_t idesc_pv = Sh::FP8 ? idesc_e4m3_f32(128, Sh::MN, true, true)
                                              : idesc_bf16_f32(128, NP, true, true);
        uint32_t pi = it;
        bool ok = true;
        for (int si = 0; si < nseg && ok; ++si) {
          const Segment sg = segs[si];
          for (int t = sg.tile_begin; t < sg.tile_end; ++t, ++pi) {
            ok = mbar_wait(&pfull_bar[pi % Sh::PR], (pi / Sh::PR) & 1, abort_flag, p.wait_limit_ns);
            MLRA_TRACE_POINT(1, 464 + min((int)pi, 31));
            if (!ok) break;
            tc_fence_after();
            MLRA_TRACE_POINT(1, 72 + min((int)pi, 31));
            const bool first = t == sg.tile_begin;
            const uint32_t st_addr = smem_u32(stages + tile_slot<Sh>(pi) * Sh::STAGE_BYTES);
            // the stage is freed after its last tile (or the launch's last tile)
            const bool frees = pi % Sh::TPS == Sh::TPS - 1 || (!more && si == nseg - 1 && t == sg.tile_end - 1);
            const uint32_t p_addr = Sh::P_IN_STAGE ? st_addr + Sh::NC * Sh::C_REG
                                                   : smem_u32(pbufs + (pi % max(Sh::PBUF, 1)) * Sh::P_BYTES);
#pragma unroll
            for (int mt = 0; mt < Sh::NMT; ++mt) {
#pragma unroll
              for (int ks = 0; ks < kTile / Sh::KT; ++ks) {
                const uint64_t a = smem_desc(st_addr + mt * (128 / Sh::CW) * Sh::C_REG + ks * Sh::KT * Sh::C_ROWB,
                                             Sh::PV_LBO, 8 * Sh::C_ROWB, swizzle_code(Sh::C_ROWB));
                const uint64_t b = smem_desc(p_addr + ks * Sh::KT * Sh::P_ROWB, Sh::P_BYTES, 8 * Sh::P_ROWB,
                                             swizzle_code(Sh::P_ROWB));
                shape_mma<Sh>(tbase + Sh::O_COL + mt * Sh::MN, a, b, idesc_pv, (first && ks == 0) ? 0u : 1u);
              }
              // this M tile's columns are read: its group may be reloaded (the last group also
              // holds the RoPE columns and P, read by every M tile)
              if (frees) umma_commit(&empty_bar[tile_stage<Sh>(pi) * Sh::NG + mt]);
            }
            umma_commit(&pvdone_bar[pi % Sh::PR]);
          }
        }
      }
      __syncwarp();
      uint32_t list_tiles = 0;
      for (int i = 0; i < nseg; ++i) list_tiles += segs[i].tile_end - segs[i].tile_begin;
      it += list_tiles;
    } else {
      // ============================== softmax / epilogue ==============================
      // NWG warpgroups, each owning HW of the CTA's heads (S^T / O^T columns and P bytes of
      // its own). Within a warpgroup the four warps take every decision together: a failed
      // wait in any of them is folded into a 128-thread OR barrier before anyone leaves, so no
      // warp is left waiting on a named barrier the others never reach.
      constexpr int HW = Sh::HW;
      const int g = (warp - 2) >> 2;      // warpgroup
      const int sw = (warp - 2) & 3;      // warp within the group
      const int q4 = warp & 3;            // TMEM lane quadrant this warp may access
      const int row = q4 * 32 + lane;     // token row of S^T, feature row of O^T
      const int hcol = g * HW;            // first head column of this warpgroup
      const int bar_or = 1 + 2 * g, bar_sync = 2 + 2 * g;
      const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
      float* red = red_sm + g * 4 * HW;
      // running max per head (shared memory or registers, see DecodeShape::M_SMEM)
      float m_reg[Sh::M_SMEM ? 1 : HW];
      float* m_sm = reinterpret_cast<float*>(smem + Sh::OFF_M) + (warp - 2) * HW;
      auto m = [&](int x) -> float& { return Sh::M_SMEM ? m_sm[x] : m_reg[x % (Sh::M_SMEM ? 1 : HW)]; };
      // E4M3 cache: each head's query terms carry a power-of-two factor (absorb kernel), read
      // from the workspace once per segment; the absorb kernel must have finished writing it
      float qf[Sh::FP8 ? HW : 1];
      if constexpr (Sh::FP8) grid_dependency_wait();
      bool ok = true;
      for (int si = 0; si < nseg && ok; ++si) {
        const Segment sg = segs[si];
        const int slot = sg.b + group;
        if constexpr (Sh::FP8) {
          const float4* fsrc = reinterpret_cast<const float4*>(p.qfac + ((size_t)sg.b * p.nsub + sub) * NP + hcol);
#pragma unroll
          for (int x = 0; x < HW; x += 4) {
            const float4 f = __ldg(fsrc + x / 4);
            qf[x] = f.x; qf[x + 1] = f.y; qf[x + 2] = f.z; qf[x + 3] = f.w;
          }
        }
        for (int t = sg.tile_begin; t < sg.tile_end; ++t, ++it) {
          const bool first = (t == sg.tile_begin);
          const bool last = (t == sg.tile_end - 1);
          const bool tile_full = (t + 1) * kTile <= sg.n;
          const bool valid = t * kTile + row < sg.n;
          bool okl = mbar_wait(&sfull_bar[it % Sh::SBUF], (it / Sh::SBUF) & 1, abort_flag, p.wait_limit_ns);
          if (!Sh::P_IN_STAGE && it >= Sh::PBUF) {  // the PV that last read this P buffer must be done
            const uint32_t j = it - Sh::PBUF;
            okl = okl && mbar_wait(&pvdone_bar[j % Sh::PR], (j / Sh::PR) & 1, abort_flag, p.wait_limit_ns);
          }
          if (warp == 2 && lane == 0) MLRA_TRACE_POINT(1, 104 + min((int)it, 31));
          if (warp == 6 && lane == 0) MLRA_TRACE_POINT(1, 320 + min((int)it, 31));
          tc_fence_after();
          float s[HW];
          const uint32_t s_addr = tbase + lane_base + Sh::S_COL0 + (it % Sh::SBUF) * Sh::MN + hcol;
          tmem_load_row<HW>(s_addr, s);
          if constexpr (Sh::FP8) {
            // score = factor * (S from the hi terms + S from the lo terms)
            float s_lo[HW];
            tmem_load_row<HW>(s_addr + NP, s_lo);
            tmem_ld_wait();
#pragma unroll
            for (int x = 0; x < HW; ++x) s[x] = (s[x] + s_lo[x]) * qf[x];
          } else {
            tmem_ld_wait();
          }
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sfree_bar[it % Sh::SBUF]);

          if (first) {
            // baseline 0 until the segment's first tile maximum is known, so that xs below
            // holds the scores themselves
            if constexpr (Sh::M_SMEM) {
              __syncwarp();
              for (int x = lane; x < HW; x += 32) m_sm[x] = 0.f;
              __syncwarp();
            } else {
#pragma unroll
              for (int x = 0; x < HW; ++x) m(x) = 0.f;
            }
          }
          // Common case: scores relative to the running max, exp2 issued before the vote. The
          // raw scores are not kept: where the rare rescale path needs them it takes xs + m.
          float xs[HW];
#pragma unroll
          for (int x = 0; x < HW; x += 2) sub_f32x2(xs[x], xs[x + 1], s[x], s[x + 1], m(x), m(x + 1));
          if (!tile_full && !valid) {
#pragma unroll
            for (int x = 0; x < HW; ++x) xs[x] = -INFINITY;
          }
          static_assert(HW % 4 == 0, "four max chains");
          float d0 = xs[0], d1 = xs[1], d2 = xs[2], d3 = xs[3];
#pragma unroll
          for (int x = 4; x < HW; x += 4) {
            d0 = fmaxf(d0, xs[x]);
            d1 = fmaxf(d1, xs[x + 1]);
            d2 = fmaxf(d2, xs[x + 2]);
            d3 = fmaxf(d3, xs[x + 3]);
          }
          const float dmax = fmaxf(fmaxf(d0, d1), fmaxf(d2, d3));
          float pr[HW];
#pragma unroll
          for (int x = 0; x < HW; ++x) pr[x] = fast_exp2(xs[x]);

          const bool need = named_bar_or(bar_or, 128, !okl || first || dmax > Sh::SLACK);
          if (warp == 2 && lane == 0) MLRA_TRACE_POINT(1, 256 + min((int)it, 31));
          if (need) {
            if (named_bar_or(bar_or, 128, !okl || *abort_flag)) { ok = false; break; }
            float tmax[HW];
#pragma unroll
            for (int x = 0; x < HW; ++x) tmax[x] = valid ? xs[x] + m(x) : -INFINITY;
            warp_reduce_scatter<HW, true>(tmax, lane);
            store_scattered<HW>(tmax, red + q4 * HW, lane);
            named_bar_sync(bar_sync, 128);
            float alpha[HW];
#pragma unroll
            for (int x = 0; x < HW; ++x) {
              const float tm = fmaxf(fmaxf(red[x], red[HW + x]), fmaxf(red[2 * HW + x], red[3 * HW + x]));
              const float mo = m(x);
              const float mn = first ? tm : fmaxf(mo, tm);
              alpha[x] = first ? 0.f : fast_exp2(mo - mn);
              pr[x] = valid ? fast_exp2((xs[x] + mo) - mn) : 0.f;
              if constexpr (!Sh::M_SMEM) m(x) = mn;
            }
            if constexpr (Sh::M_SMEM) {
              // raise the warp's copy once every lane has read the old values (red stays intact
              // until the barrier below)
              __syncwarp();
              for (int x = lane; x < HW; x += 32) {
                const float tm = fmaxf(fmaxf(red[x], red[HW + x]), fmaxf(red[2 * HW + x], red[3 * HW + x]));
                m_sm[x] = first ? tm : fmaxf(m_sm[x], tm);
              }
              __syncwarp();
            }
#pragma unroll
            for (int x = 0; x < HW; ++x) l_part[x] = first ? 0.f : l_part[x] * alpha[x];
            if (!first) {
              // O holds the sums up to tile it-1: wait for that PV, then rescale its columns
              const bool okr = mbar_wait(&pvdone_bar[(it - 1) % Sh::PR], ((it - 1) / Sh::PR) & 1, abort_flag,
                                         p.wait_limit_ns);
              if (named_bar_or(bar_or, 128, !okr)) { ok = false; break; }
              tc_fence_after();
#pragma unroll
              for (int mt = 0; mt < Sh::NMT; ++mt) {
#pragma unroll
                for (int qt = 0; qt < Sh::NQ; ++qt) {  // every term's columns
                  float o[HW];
                  const uint32_t oa = tbase + lane_base + Sh::O_COL + mt * Sh::MN + qt * NP + hcol;
                  tmem_load_row<HW>(oa, o);
                  tmem_ld_wait();
#pragma unroll
                  for (int x = 0; x < HW; ++x) o[x] *= alpha[x];
                  tmem_store_row<HW>(oa, o);
                }
              }
              tmem_st_wait();
            }
            named_bar_sync(bar_sync, 128);  // everyone has read red
          }
#pragma unroll
          for (int x = 0; x < HW; x += 2)
            add_f32x2(l_part[x], l_part[x + 1], l_part[x], l_part[x + 1], pr[x], pr[x + 1]);
          uint8_t* pbuf = Sh::P_IN_STAGE ? stages + tile_slot<Sh>(it) * Sh::STAGE_BYTES + Sh::NC * Sh::C_REG
                                         : pbufs + (it % max(Sh::PBUF, 1)) * Sh::P_BYTES;
          if constexpr (Sh::FP8) {
            // P row = [hi terms of the NP heads | lo terms], E4M3, of p * P_SCALE; 8 heads per
            // 8-byte store (a swizzle moves whole 16-byte chunks, so 8 aligned bytes stay together)
#pragma unroll
            for (int c = 0; c < HW / 8; ++c) {
              uint32_t hw[2], lw[2];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                uint16_t h2, l2;
                e4m3x2_split(pr[8 * c + 2 * e] * Sh::P_SCALE, pr[8 * c + 2 * e + 1] * Sh::P_SCALE, h2, l2);
                if (e % 2 == 0) {
                  hw[e / 2] = h2;
                  lw[e / 2] = l2;
                } else {
                  hw[e / 2] |= static_cast<uint32_t>(h2) << 16;
                  lw[e / 2] |= static_cast<uint32_t>(l2) << 16;
                }
              }
              *reinterpret_cast<uint2*>(pbuf + swizzle(row * Sh::P_ROWB + hcol + c * 8, Sh::P_ROWB)) =
                  make_uint2(hw[0], hw[1]);
              *reinterpret_cast<uint2*>(pbuf + swizzle(row * Sh::P_ROWB + NP + hcol + c * 8, Sh::P_ROWB)) =
                  make_uint2(lw[0], lw[1]);
            }
          } else {
#pragma unroll
            for (int c = 0; c < HW / 8; ++c) {
              uint4 w;
              w.x = pack_bf16x2(pr[8 * c + 0], pr[8 * c + 1]);
              w.y = pack_bf16x2(pr[8 * c + 2], pr[8 * c + 3]);
              w.z = pack_bf16x2(pr[8 * c + 4], pr[8 * c + 5]);
              w.w = pack_bf16x2(pr[8 * c + 6], pr[8 * c + 7]);
              *reinterpret_cast<uint4*>(pbuf + swizzle(row * Sh::P_ROWB + hcol * 2 + c * 16, Sh::P_ROWB)) = w;
            }
          }
          if (g == 0 && last && !valid) {
            // rows past the sequence end: zero them so stale or NaN slots cannot reach O
            uint8_t* st = stages + tile_slot<Sh>(it) * Sh::STAGE_BYTES;
#pragma unroll
            for (int r = 0; r < Sh::NC; ++r)
#pragma unroll
              for (int c = 0; c < Sh::C_ROWB / 16; ++c)
                *reinterpret_cast<uint4*>(st + r * Sh::C_REG + row * Sh::C_ROWB + c * 16) =
                    make_uint4(0, 0, 0, 0);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&pfull_bar[it % Sh::PR]);
          if (warp == 2 && lane == 0) MLRA_TRACE_POINT(1, 136 + min((int)it, 31));
          if (warp == 6 && lane == 0) MLRA_TRACE_POINT(1, 288 + min((int)it, 31));

          if (last) {
            // ---- segment epilogue: O / l and lse of this warpgroup's heads ----
            const bool oke = mbar_wait(&pvdone_bar[it % Sh::PR], (it / Sh::PR) & 1, abort_flag, p.wait_limit_ns);
            if (named_bar_or(bar_or, 128, !oke || *abort_flag)) { ok = false; ++it; break; }
            tc_fence_after();
            float lt[HW];
#pragma unroll
            for (int x = 0; x < HW; ++x) lt[x] = l_part[x];
            warp_reduce_scatter<HW, false>(lt, lane);
            store_scattered<HW>(lt, red + q4 * HW, lane);
            named_bar_sync(bar_sync, 128);
            // This runs while the next segment's tiles wait behind it, so it is kept short: 1 / l
            // by an approximate reciprocal (l >= 1: the running maximum's own term contributes 1,
            // so the 2-ulp bound of div.approx holds), and each warp stores its lse values with
            // one instruction, lane x holding head x.
            if constexpr (HW >= 32 && Sh::NMT == 1) {
              // 32 heads per warpgroup and one O tile: lane x of every warp works out head x's
              // 1 / l and lse, and the O rows take 1 / l by shuffle (measured faster than every
              // thread computing all 32; with several O tiles it is not)
              static_assert(HW <= 32, "one lane per head");
              float inv_lane = 0.f, lse_lane = 0.f;
              {
                float mv = 0.f;
#pragma unroll
                for (int x = 0; x < HW; ++x)
                  if (x == lane) mv = m(x);
                if (lane < HW) {
                  const float l = red[lane] + red[HW + lane] + red[2 * HW + lane] + red[3 * HW + lane];
                  inv_lane = __fdividef(Sh::FP8 ? p.o_scale : 1.f, l);
                  lse_lane = mv + __log2f(l);
                }
              }
              if (sw == 0 && lane < HW && hcol + lane < nheads)
                p.lse_part[(size_t)slot * p.h + head0 + hcol + lane] = lse_lane;
#pragma unroll
              for (int mt = 0; mt < Sh::NMT; ++mt) {
                float o[HW];
                tmem_load_row<HW>(tbase + lane_base + Sh::O_COL + mt * Sh::MN + hcol, o);
                if constexpr (Sh::FP8) {
                  float o_lo[HW];
                  tmem_load_row<HW>(tbase + lane_base + Sh::O_COL + mt * Sh::MN + NP + hcol, o_lo);
                  tmem_ld_wait();
#pragma unroll
                  for (int x = 0; x < HW; ++x) o[x] += o_lo[x];
                } else {
                  tmem_ld_wait();
                }
                const int f = mt * 128 + row;
                float* dst = p.o_part + ((size_t)slot * p.h + head0 + hcol) * Sh::DB + f;
#pragma unroll
                for (int x = 0; x < HW; ++x) {
                  const float ix = __shfl_sync(0xffffffffu, inv_lane, x);
                  if (f < Sh::DB && hcol + x < nheads) dst[(size_t)x * Sh::DB] = o[x] * ix;
                }
              }
            } else {
              // otherwise every thread works out 1 / l of each head itself
              static_assert(HW <= 32, "one lse lane per head");
              float inv[HW];
              float lse_lane = 0.f;
#pragma unroll
              for (int x = 0; x < HW; ++x) {
                const float l = red[x] + red[HW + x] + red[2 * HW + x] + red[3 * HW + x];
                inv[x] = __fdividef(Sh::FP8 ? p.o_scale : 1.f, l);
                if (x == lane) lse_lane = m(x) + __log2f(l);
              }
              if (sw == 0 && lane < HW && hcol + lane < nheads)
                p.lse_part[(size_t)slot * p.h + head0 + hcol + lane] = lse_lane;
#pragma unroll
              for (int mt = 0; mt < Sh::NMT; ++mt) {
                float o[HW];
                tmem_load_row<HW>(tbase + lane_base + Sh::O_COL + mt * Sh::MN + hcol, o);
                if constexpr (Sh::FP8) {
                  float o_lo[HW];
                  tmem_load_row<HW>(tbase + lane_base + Sh::O_COL + mt * Sh::MN + NP + hcol, o_lo);
                  tmem_ld_wait();
#pragma unroll
                  for (int x = 0; x < HW; ++x) o[x] += o_lo[x];
                } else {
                  tmem_ld_wait();
                }
                const int f = mt * 128 + row;
                if (f < Sh::DB) {
                  float* dst = p.o_part + ((size_t)slot * p.h + head0 + hcol) * Sh::DB + f;
#pragma unroll
                  for (int x = 0; x < HW; ++x)
                    if (hcol + x < nheads) dst[(size_t)x * Sh::DB] = o[x] * inv[x];
                }
              }
            }
            tc_fence_before();
            named_bar_sync(bar_sync, 128);  // red and O reads are done before the next segment
            if (warp == 2 && lane == 0) MLRA_TRACE_POINT(1, 168 + min(si, 7));
          }
        }
      }
    }
    __syncthreads();
    if (*abort_flag) break;
  }

  if (threadIdx.x == 0) MLRA_TRACE_POINT(1, 200);
  // ---- teardown: nothing may be in flight when shared memory and TMEM are released ----
  if (warp == 0 && lane == 0) {
    // wait for the last issued load of every (stage, group) (completed loads return at once)
    for (int gi = 0; gi < STAGES * Sh::NG; ++gi) {
      if (!(issued_mask & (1u << gi))) continue;
      if (!mbar_wait_drain(&full_bar[gi], (issued_phase >> gi) & 1, p.wait_limit_ns)) *drain_err = 1;
    }
  }
  if (warp == 1 || warp == Sh::PV_WARP) {
    uint64_t* done = &mmadone_bar[warp == 1 ? 0 : 1];
    if (lane == 0) umma_commit(done);
    __syncwarp();
    if (!mbar_wait_drain(done, 0, p.wait_limit_ns) && lane == 0) *drain_err = 1;
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    // Every CTA waits for the absorb kernel before it exits (a CTA without tiles never did),
    // so this grid completes only after the absorb grid, and the status word it cleared is
    // not written by this call's later kernels before the clear.
    grid_dependency_wait();
    if (blockIdx.x == 0) fold_early(p.tags, p.status);
    if (*abort_flag) set_status(p.status, kErrTimeout);
    if (*drain_err) force_status(p.status, kErrDrain);
  }
  if (threadIdx.x == 0) MLRA_TRACE_POINT(1, 201);
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, Sh::TMEM_COLS);
  }
}

}  // namespace mlra
