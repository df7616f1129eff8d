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
// Roles (192 threads): warp 0 issues TMA loads of pages and queries, warp 1 allocates TMEM
// and issues the MMAs, warps 2..5 run the softmax and write the partial results. They
// hand off through mbarriers; each wait is bounded (see mbar_wait).
//
// Softmax detail: each thread owns one token row of S^T and all its heads. The running
// maximum m_h is only raised when some score exceeds it by more than kRescaleSlack (in
// log2 units); otherwise P = exp2(s - m_h) is used as is (values up to 2^slack are exact in
// fp32/bf16 range). A raise costs a cross-thread max and a rescale of O in TMEM; it happens
// on a segment's first tile and then rarely.
#pragma once

#include "common.cuh"

namespace mlra {

constexpr float kRescaleSlack = 8.0f;

__host__ __device__ constexpr int round_up(int x, int m) { return (x + m - 1) / m * m; }

template <int DB_, int DR_, int NP_, int STAGES_, int QBUF_, int PBUF_>
struct DecodeShape {
  static constexpr int DB = DB_;      // latent block width d_c / k
  static constexpr int DR = DR_;      // RoPE key width
  static constexpr int NP = NP_;      // heads per CTA (MMA N), 16 / 32 / 64
  static constexpr int STAGES = STAGES_;
  static constexpr int QBUF = QBUF_;  // query buffers
  static constexpr int PBUF = PBUF_;  // probability buffers
  // A cache row is split into swizzle-width regions: block columns and RoPE columns.
  static constexpr int CW = DB < 64 ? DB : 64;
  static constexpr int NC = DB / CW;
  static constexpr int RW = DR < 64 ? DR : 64;
  static constexpr int NR = DR / RW;
  static constexpr int C_ROWB = CW * 2;
  static constexpr int R_ROWB = RW * 2;
  static constexpr int C_REG = round_up(kTile * C_ROWB, 1024);
  static constexpr int R_REG = round_up(kTile * R_ROWB, 1024);
  static constexpr int STAGE_BYTES = NC * C_REG + NR * R_REG;
  static constexpr int PAGE_TX = NC * kPage * C_ROWB + NR * kPage * R_ROWB;
  static constexpr int QC_REG = round_up(NP * C_ROWB, 1024);
  static constexpr int QR_REG = round_up(NP * R_ROWB, 1024);
  static constexpr int Q_BYTES = NC * QC_REG + NR * QR_REG;
  static constexpr int Q_TX = NP * (DB + DR) * 2;
  static constexpr int P_ROWB = NP * 2;
  static constexpr int P_BYTES = round_up(kTile * P_ROWB, 1024);
  static constexpr int NMT = DB >= 128 ? DB / 128 : 1;  // PV M tiles
  static constexpr uint32_t PV_LBO = DB >= 128 ? C_REG : 0;  // next 64-feature chunk
  static constexpr int S_COL0 = 0;                  // two S buffers of NP columns
  static constexpr int O_COL = 2 * NP;              // NMT x NP columns
  static constexpr int TMEM_USED = 2 * NP + NMT * NP;
  static constexpr int TMEM_COLS = TMEM_USED <= 32 ? 32 : TMEM_USED <= 64 ? 64 :
                                   TMEM_USED <= 128 ? 128 : TMEM_USED <= 256 ? 256 : 512;
  static constexpr int MAX_SEGS = 64;
  // small shared state after the big buffers
  static constexpr int OFF_STAGES = 0;
  static constexpr int OFF_Q = OFF_STAGES + STAGES * STAGE_BYTES;
  static constexpr int OFF_P = OFF_Q + QBUF * Q_BYTES;
  static constexpr int OFF_M = OFF_P + PBUF * P_BYTES;          // NP floats
  static constexpr int OFF_RED = OFF_M + NP * 4;                // 4 x NP floats
  static constexpr int OFF_SEG = OFF_RED + 4 * NP * 4;          // MAX_SEGS segments
  static constexpr int OFF_BAR = round_up(OFF_SEG + MAX_SEGS * 16, 8);
  static constexpr int NUM_BARS = 2 * STAGES + 2 * QBUF + 8 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NUM_BARS * 8;       // tmem slot, flags, scratch
  static constexpr int SMEM_BYTES = OFF_MISC + 64 * 4 + 1024;  // + alignment slack
  static_assert(DB % CW == 0 && DR % RW == 0, "region split");
  static_assert(NP == 16 || NP == 32 || NP == 64, "heads per CTA");
  static_assert(QBUF == 1 || QBUF == 2, "query buffers");
  static_assert(PBUF == 1 || PBUF == 2, "P buffers");
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
  float* o_part;    // [slots][h][DB] fp32, normalised partial latent outputs
  float* lse_part;  // [slots][h] fp32, log2-domain log-sum-exp
  int* status;
  unsigned long long wait_limit_ns;
  int inject_stall;  // test hook: the producer withholds its first tile
};

// Reduce NP values across the 32 lanes of a warp and scatter the results: afterwards lane l
// holds in v[0..max(1, NP/32)) the reduction of heads [l*NP/32, (l+1)*NP/32) (NP >= 32) or of
// head (l & 15) (NP == 16).
template <bool IS_MAX>
__device__ __forceinline__ float red_op(float a, float b) {
  return IS_MAX ? fmaxf(a, b) : a + b;
}
template <int OFF, int N, bool IS_MAX, int NP>
__device__ __forceinline__ void rs_step(float (&v)[NP], int lane) {
  const bool upper = (lane & OFF) != 0;
#pragma unroll
  for (int x = 0; x < N / 2; ++x) {
    const float send = upper ? v[x] : v[x + N / 2];
    const float keep = upper ? v[x + N / 2] : v[x];
    v[x] = red_op<IS_MAX>(keep, __shfl_xor_sync(0xffffffffu, send, OFF));
  }
}
template <int NP, bool IS_MAX>
__device__ __forceinline__ void warp_reduce_scatter(float (&v)[NP], int lane) {
  if constexpr (NP == 16) {
#pragma unroll
    for (int x = 0; x < 16; ++x) v[x] = red_op<IS_MAX>(v[x], __shfl_xor_sync(0xffffffffu, v[x], 16));
    rs_step<8, 16, IS_MAX>(v, lane);
    rs_step<4, 8, IS_MAX>(v, lane);
    rs_step<2, 4, IS_MAX>(v, lane);
    rs_step<1, 2, IS_MAX>(v, lane);
  } else {
    rs_step<16, NP, IS_MAX>(v, lane);
    rs_step<8, NP / 2, IS_MAX>(v, lane);
    rs_step<4, NP / 4, IS_MAX>(v, lane);
    rs_step<2, NP / 8, IS_MAX>(v, lane);
    rs_step<1, NP / 16, IS_MAX>(v, lane);
  }
}
// Writes the scattered per-head values of this lane to dst[h].
template <int NP>
__device__ __forceinline__ void store_scattered(const float (&v)[NP], float* dst, int lane) {
  if constexpr (NP == 16) {
    if (lane < 16) dst[lane] = v[0];
  } else {
#pragma unroll
    for (int x = 0; x < NP / 32; ++x) dst[lane * (NP / 32) + x] = v[x];
  }
}

template <class Sh>
__global__ void __launch_bounds__(192, 1)
    mlra_decode_kernel(const __grid_constant__ CUtensorMap map_c,
                       const __grid_constant__ CUtensorMap map_r,
                       const __grid_constant__ CUtensorMap map_qc,
                       const __grid_constant__ CUtensorMap map_qr, const DecodeParams p) {
  constexpr int NP = Sh::NP, STAGES = Sh::STAGES;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* stages = smem + Sh::OFF_STAGES;
  uint8_t* qbufs = smem + Sh::OFF_Q;
  uint8_t* pbufs = smem + Sh::OFF_P;
  float* m_sm = reinterpret_cast<float*>(smem + Sh::OFF_M);
  float* red_sm = reinterpret_cast<float*>(smem + Sh::OFF_RED);
  Segment* segs = reinterpret_cast<Segment*>(smem + Sh::OFF_SEG);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sh::OFF_BAR);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* qfull_bar = bars + 2 * STAGES;
  uint64_t* qempty_bar = qfull_bar + Sh::QBUF;
  uint64_t* sfull_bar = qempty_bar + Sh::QBUF;
  uint64_t* sfree_bar = sfull_bar + 2;
  uint64_t* pfull_bar = sfree_bar + 2;
  uint64_t* pvdone_bar = pfull_bar + 2;
  uint64_t* mmadone_bar = pvdone_bar + 2;
  int* misc = reinterpret_cast<int*>(smem + Sh::OFF_MISC);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc);
  volatile int* abort_flag = misc + 1;
  int* plan_err = misc + 2;
  int* scratch = misc + 8;  // 40 ints for the planner

  const int warp = warp_id(), lane = lane_id();
  const int group = blockIdx.x / p.nsub;
  const int sub = blockIdx.x % p.nsub;
  const int blk = sub / p.chunks;
  const int chunk = sub % p.chunks;
  const int head0 = blk * p.heads_block + chunk * NP;
  const int nheads = min(NP, p.heads_block - chunk * NP);
  const int cap_len = p.pt_stride * kPage;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full_bar[s], 1);
      mbar_init(&empty_bar[s], 1);
    }
    for (int s = 0; s < Sh::QBUF; ++s) {
      mbar_init(&qfull_bar[s], 1);
      mbar_init(&qempty_bar[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&sfull_bar[s], 1);
      mbar_init(&sfree_bar[s], 4);
      mbar_init(&pfull_bar[s], 4);
      mbar_init(&pvdone_bar[s], 1);
    }
    mbar_init(mmadone_bar, 1);
    *abort_flag = 0;
    *plan_err = 0;
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
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  // ---- plan: which flattened tiles this group owns (seq_lens do not depend on the
  // previous kernel, so this overlaps its tail under programmatic dependent launch) ----
  int err = 0;
  const int T = block_total_tiles(p.seq_lens, p.batch, cap_len, scratch, &err);
  const int quota = T > 0 ? (T + p.groups - 1) / p.groups : 1;
  const int lo = min(group * quota, T);
  const int hi = min(lo + quota, T);
  if (err) atomicOr(plan_err, 1);

  // pipeline counters persist across segment-list refills
  uint32_t it = 0;      // tiles consumed/produced so far by this role
  uint32_t segc = 0;    // segments so far
  // MMA-role state of the previous tile (its PV is issued one tile late)
  bool prev_valid = false, prev_first = false;
  uint32_t prev_it = 0;
  // producer: last issued phase per stage, for the drain at the end
  uint32_t issued_mask = 0;
  // softmax-role partial sums
  float l_part[NP];
#pragma unroll
  for (int x = 0; x < NP; ++x) l_part[x] = 0.f;

  int b_start = 0, p_start = 0;
  bool more = lo < hi;
  while (more) {
    int more_i, rb, rp;
    const int nseg = block_collect_segments(p.seq_lens, p.batch, cap_len, lo, hi, b_start, p_start,
                                            segs, Sh::MAX_SEGS, scratch, &more_i, &rb, &rp, &err);
    more = more_i != 0;
    b_start = rb;
    p_start = rp;

    if (warp == 0) {
      // ============================== TMA producer ==============================
      const uint64_t pol_stream = l2_policy_evict_first();
      const uint64_t pol_keep = l2_policy_evict_last();
      grid_dependency_wait();  // q_pack and the reset status word come from the absorb kernel
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
            mbar_arrive_expect_tx(&qfull_bar[qb], Sh::Q_TX);
            const int qrow = (sg.b * p.nsub + sub) * NP;
            for (int r = 0; r < Sh::NC; ++r)
              tma_load_2d(qdst + r * Sh::QC_REG, &map_qc, &qfull_bar[qb], r * Sh::CW, qrow, pol_keep);
            for (int r = 0; r < Sh::NR; ++r)
              tma_load_2d(qdst + Sh::NC * Sh::QC_REG + r * Sh::QR_REG, &map_qr, &qfull_bar[qb],
                          Sh::DB + r * Sh::RW, qrow, pol_keep);
          }
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        ++segc;
        int pbase = -64, pid = 0;
        for (int t = sg.tile_begin; t < sg.tile_end; ++t, ++it) {
          const int p0 = 2 * t;
          if (p0 + 1 >= pbase + 32) {
            pbase = p0;
            const int pp = pbase + lane;
            pid = pp < pages_b ? __ldg(p.page_table + (size_t)sg.b * p.pt_stride + pp) : 0;
          }
          int id0 = __shfl_sync(0xffffffffu, pid, p0 - pbase);
          int id1 = __shfl_sync(0xffffffffu, pid, p0 + 1 - pbase);
          const int npg = (p0 + 1 < pages_b) ? 2 : 1;
          ok = true;
          if (lane == 0) {
            if (id0 < 0 || id0 >= p.num_pages) { set_status(p.status, kErrPageOob); id0 = 0; }
            if (npg == 2 && (id1 < 0 || id1 >= p.num_pages)) { set_status(p.status, kErrPageOob); id1 = 0; }
            const int st = it % STAGES;
            ok = mbar_wait(&empty_bar[st], ((it / STAGES) & 1) ^ 1, abort_flag, p.wait_limit_ns);
            if (ok && !(p.inject_stall && it == 0)) {
              uint8_t* dst = stages + st * Sh::STAGE_BYTES;
              mbar_arrive_expect_tx(&full_bar[st], npg * Sh::PAGE_TX);
              issued_mask |= 1u << st;
              for (int pg = 0; pg < npg; ++pg) {
                const int y = (pg ? id1 : id0) * kPage;
                for (int r = 0; r < Sh::NC; ++r)
                  tma_load_2d(dst + r * Sh::C_REG + pg * kPage * Sh::C_ROWB, &map_c, &full_bar[st],
                              blk * Sh::DB + r * Sh::CW, y, pol_stream);
                for (int r = 0; r < Sh::NR; ++r)
                  tma_load_2d(dst + Sh::NC * Sh::C_REG + r * Sh::R_REG + pg * kPage * Sh::R_ROWB,
                              &map_r, &full_bar[st], p.d_c + r * Sh::RW, y, pol_keep);
              }
            }
          }
          if (!__shfl_sync(0xffffffffu, ok, 0)) break;
        }
      }
    } else if (warp == 1) {
      // ============================== MMA issuer ==============================
      constexpr uint32_t idesc_qk = idesc_bf16_f32(128, NP, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(128, NP, true, true);
      auto issue_pv = [&](uint32_t j, bool first) -> bool {
        bool ok = mbar_wait(&pfull_bar[j & 1], (j >> 1) & 1, abort_flag, p.wait_limit_ns);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) return false;
        tc_fence_after();
        if (lane == 0) {
          const uint32_t st_addr = smem_u32(stages + (j % STAGES) * Sh::STAGE_BYTES);
          const uint32_t p_addr = smem_u32(pbufs + (j % Sh::PBUF) * Sh::P_BYTES);
#pragma unroll
          for (int mt = 0; mt < Sh::NMT; ++mt) {
#pragma unroll
            for (int ks = 0; ks < kTile / 16; ++ks) {
              const uint64_t a = smem_desc(st_addr + mt * (128 / Sh::CW) * Sh::C_REG + ks * 16 * Sh::C_ROWB,
                                           Sh::PV_LBO, 8 * Sh::C_ROWB, swizzle_code(Sh::C_ROWB));
              const uint64_t b = smem_desc(p_addr + ks * 16 * Sh::P_ROWB, Sh::P_BYTES,
                                           8 * Sh::P_ROWB, swizzle_code(Sh::P_ROWB));
              umma_bf16(tbase + Sh::O_COL + mt * NP, a, b, idesc_pv, (first && ks == 0) ? 0u : 1u);
            }
          }
          umma_commit(&empty_bar[j % STAGES]);
          umma_commit(&pvdone_bar[j & 1]);
        }
        __syncwarp();
        return true;
      };
      bool ok = true;
      for (int si = 0; si < nseg && ok; ++si) {
        const Segment sg = segs[si];
        const int qb = segc % Sh::QBUF;
        ok = __all_sync(0xffffffffu, mbar_wait(&qfull_bar[qb], (segc / Sh::QBUF) & 1, abort_flag,
                                               p.wait_limit_ns));
        if (!ok) break;
        const uint32_t q_addr = smem_u32(qbufs + qb * Sh::Q_BYTES);
        for (int t = sg.tile_begin; t < sg.tile_end && ok; ++t, ++it) {
          const int st = it % STAGES;
          ok = mbar_wait(&full_bar[st], (it / STAGES) & 1, abort_flag, p.wait_limit_ns);
          if (ok && it >= 2)
            ok = mbar_wait(&sfree_bar[it & 1], ((it >> 1) - 1) & 1, abort_flag, p.wait_limit_ns);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
          if (lane == 0) {
            const uint32_t st_addr = smem_u32(stages + st * Sh::STAGE_BYTES);
            const uint32_t d = tbase + Sh::S_COL0 + (it & 1) * NP;
            uint32_t acc = 0;
#pragma unroll
            for (int r = 0; r < Sh::NC; ++r) {
#pragma unroll
              for (int ks = 0; ks < Sh::C_ROWB / 32; ++ks) {
                const uint64_t a = smem_desc(st_addr + r * Sh::C_REG + ks * 32, 16, 8 * Sh::C_ROWB,
                                             swizzle_code(Sh::C_ROWB));
                const uint64_t b = smem_desc(q_addr + r * Sh::QC_REG + ks * 32, 16, 8 * Sh::C_ROWB,
                                             swizzle_code(Sh::C_ROWB));
                umma_bf16(d, a, b, idesc_qk, acc);
                acc = 1;
              }
            }
#pragma unroll
            for (int r = 0; r < Sh::NR; ++r) {
#pragma unroll
              for (int ks = 0; ks < Sh::R_ROWB / 32; ++ks) {
                const uint64_t a = smem_desc(st_addr + Sh::NC * Sh::C_REG + r * Sh::R_REG + ks * 32, 16,
                                             8 * Sh::R_ROWB, swizzle_code(Sh::R_ROWB));
                const uint64_t b = smem_desc(q_addr + Sh::NC * Sh::QC_REG + r * Sh::QR_REG + ks * 32,
                                             16, 8 * Sh::R_ROWB, swizzle_code(Sh::R_ROWB));
                umma_bf16(d, a, b, idesc_qk, 1);
              }
            }
            umma_commit(&sfull_bar[it & 1]);
            if (t == sg.tile_end - 1) umma_commit(&qempty_bar[qb]);
          }
          __syncwarp();
          if (prev_valid) ok = issue_pv(prev_it, prev_first);
          prev_valid = true;
          prev_it = it;
          prev_first = (t == sg.tile_begin);
        }
        ++segc;
      }
      // the list's last PV (every list ends on a segment boundary)
      if (ok && prev_valid) issue_pv(prev_it, prev_first);
      prev_valid = false;
    } else {
      // ============================== softmax / epilogue ==============================
      // The four warps take every decision together: a failed wait in any of them is
      // folded into a 128-thread OR barrier before anyone leaves, so no warp is left
      // waiting on a named barrier the others never reach.
      const int sw = warp - 2;         // 0..3
      const int q4 = warp & 3;         // TMEM lane quadrant this warp may access
      const int row = q4 * 32 + lane;  // token row of S^T, feature row of O^T
      const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
      bool ok = true;
      for (int si = 0; si < nseg && ok; ++si) {
        const Segment sg = segs[si];
        const int slot = sg.b + group;
        for (int t = sg.tile_begin; t < sg.tile_end; ++t, ++it) {
          const bool first = (t == sg.tile_begin);
          const bool last = (t == sg.tile_end - 1);
          const bool valid = t * kTile + row < sg.n;
          bool okl = mbar_wait(&sfull_bar[it & 1], (it >> 1) & 1, abort_flag, p.wait_limit_ns);
          if (it >= Sh::PBUF) {  // the PV that last read this P buffer must be done
            const uint32_t j = it - Sh::PBUF;
            okl = okl && mbar_wait(&pvdone_bar[j & 1], (j >> 1) & 1, abort_flag, p.wait_limit_ns);
          }
          tc_fence_after();
          float s[NP];
          tmem_load_row<NP>(tbase + lane_base + Sh::S_COL0 + (it & 1) * NP, s);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sfree_bar[it & 1]);

          float m[NP];
#pragma unroll
          for (int x = 0; x < NP; ++x) m[x] = first ? -INFINITY : m_sm[x];
          float dmax = -INFINITY;
          if (valid) {
#pragma unroll
            for (int x = 0; x < NP; ++x) dmax = fmaxf(dmax, s[x] - m[x]);
          }
          const bool need = named_bar_or(1, 128, !okl || first || dmax > kRescaleSlack);
          if (need) {
            if (named_bar_or(1, 128, !okl || *abort_flag)) { ok = false; break; }
            float tmax[NP];
#pragma unroll
            for (int x = 0; x < NP; ++x) tmax[x] = valid ? s[x] : -INFINITY;
            warp_reduce_scatter<NP, true>(tmax, lane);
            store_scattered<NP>(tmax, red_sm + q4 * NP, lane);
            named_bar_sync(2, 128);
            float alpha[NP];
#pragma unroll
            for (int x = 0; x < NP; ++x) {
              const float tm = fmaxf(fmaxf(red_sm[x], red_sm[NP + x]),
                                     fmaxf(red_sm[2 * NP + x], red_sm[3 * NP + x]));
              const float mn = fmaxf(m[x], tm);
              alpha[x] = first ? 0.f : fast_exp2(m[x] - mn);
              m[x] = mn;
            }
#pragma unroll
            for (int x = 0; x < NP; ++x) l_part[x] = first ? 0.f : l_part[x] * alpha[x];
            if (!first) {
              // O holds the sums up to tile it-1: wait for that PV, then rescale its columns
              const bool okr = mbar_wait(&pvdone_bar[(it - 1) & 1], ((it - 1) >> 1) & 1, abort_flag,
                                         p.wait_limit_ns);
              if (named_bar_or(1, 128, !okr)) { ok = false; break; }
              tc_fence_after();
#pragma unroll
              for (int mt = 0; mt < Sh::NMT; ++mt) {
                float o[NP];
                const uint32_t oa = tbase + lane_base + Sh::O_COL + mt * NP;
                tmem_load_row<NP>(oa, o);
                tmem_ld_wait();
#pragma unroll
                for (int x = 0; x < NP; ++x) o[x] *= alpha[x];
                tmem_store_row<NP>(oa, o);
              }
              tmem_st_wait();
            }
            named_bar_sync(2, 128);  // everyone has read red_sm and the old m_sm
            if (sw == 0) {
#pragma unroll
              for (int x = 0; x < NP; ++x)
                if (x % 32 == lane) m_sm[x] = m[x];
            }
          }
          uint8_t* pbuf = pbufs + (it % Sh::PBUF) * Sh::P_BYTES;
#pragma unroll
          for (int c = 0; c < Sh::P_ROWB / 16; ++c) {
            float pv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
              const int x = 8 * c + e;
              pv[e] = valid ? fast_exp2(s[x] - m[x]) : 0.f;
              l_part[x] += pv[e];
            }
            uint4 w;
            w.x = pack_bf16x2(pv[0], pv[1]);
            w.y = pack_bf16x2(pv[2], pv[3]);
            w.z = pack_bf16x2(pv[4], pv[5]);
            w.w = pack_bf16x2(pv[6], pv[7]);
            *reinterpret_cast<uint4*>(pbuf + swizzle(row * Sh::P_ROWB + c * 16, Sh::P_ROWB)) = w;
          }
          if (last && !valid) {
            // rows past the sequence end: zero them so stale or NaN slots cannot reach O
            uint8_t* st = stages + (it % STAGES) * Sh::STAGE_BYTES;
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
          if (lane == 0) mbar_arrive(&pfull_bar[it & 1]);
          if (need) named_bar_sync(2, 128);  // the new m_sm is visible before the next tile

          if (last) {
            // ---- segment epilogue: O / l and lse, written to the partial slot ----
            const bool oke = mbar_wait(&pvdone_bar[it & 1], (it >> 1) & 1, abort_flag, p.wait_limit_ns);
            if (named_bar_or(1, 128, !oke || *abort_flag)) { ok = false; ++it; break; }
            tc_fence_after();
            float lt[NP];
#pragma unroll
            for (int x = 0; x < NP; ++x) lt[x] = l_part[x];
            warp_reduce_scatter<NP, false>(lt, lane);
            store_scattered<NP>(lt, red_sm + q4 * NP, lane);
            named_bar_sync(2, 128);
            float inv[NP];
#pragma unroll
            for (int x = 0; x < NP; ++x) {
              const float l = red_sm[x] + red_sm[NP + x] + red_sm[2 * NP + x] + red_sm[3 * NP + x];
              inv[x] = 1.f / l;
              if (sw == 0 && x % 32 == lane && x < nheads)
                p.lse_part[(size_t)slot * p.h + head0 + x] = m[x] + __log2f(l);
            }
#pragma unroll
            for (int mt = 0; mt < Sh::NMT; ++mt) {
              float o[NP];
              tmem_load_row<NP>(tbase + lane_base + Sh::O_COL + mt * NP, o);
              tmem_ld_wait();
              const int f = mt * 128 + row;
              if (f < Sh::DB) {
                float* dst = p.o_part + ((size_t)slot * p.h + head0) * Sh::DB + f;
#pragma unroll
                for (int x = 0; x < NP; ++x)
                  if (x < nheads) dst[(size_t)x * Sh::DB] = o[x] * inv[x];
              }
            }
            tc_fence_before();
            named_bar_sync(2, 128);  // red_sm and O reads are done before the next segment
          }
        }
      }
    }
    __syncthreads();
    if (*abort_flag) break;
  }

  // ---- teardown: nothing may be in flight when shared memory and TMEM are released ----
  if (warp == 0 && lane == 0) {
    // wait for every stage's last issued load (completed loads return at once)
    for (int s = 0; s < STAGES; ++s) {
      if (!(issued_mask & (1u << s))) continue;
      // the last tile that used stage s
      const uint32_t last_it = it == 0 ? 0 : (it - 1) - ((it - 1 + STAGES - s) % STAGES);
      mbar_wait_drain(&full_bar[s], (last_it / STAGES) & 1, p.wait_limit_ns);
    }
  }
  if (warp == 1) {
    if (lane == 0) umma_commit(mmadone_bar);
    __syncwarp();
    mbar_wait_drain(mmadone_bar, 0, p.wait_limit_ns);
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) set_status(p.status, kErrTimeout);
  grid_launch_dependents();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, Sh::TMEM_COLS);
  }
}

}  // namespace mlra
