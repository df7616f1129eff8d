// proj.cuh - the two per-head projections around the latent attention kernel.
//
//   absorb:  q~_h = scale * log2(e) * (W^UK_h)^T q^C_h     (lesty.tech MLA article, section 5;
//            ai360xpert "Absorbing the up-projection"), written as bf16 into the packed query
//            [b][latent block][head][q~ | q^R] that the decode kernel streams; q^R is scaled
//            the same way, so the decode kernel's scores come out in log2 units.
//   uproj:   o_h = W^UV_h o~_h                              ("a single final matrix
//            multiplication", lesty.tech section 5), where o~_h is first merged from the
//            decode kernel's split partials by log-sum-exp.
//
// Both are one CTA per (head, batch tile): D^T[M x N] = A_h[M x K] * X_h[N x K]^T with the
// per-head weight as the tcgen05 A operand (M = 128 rows of the weight's output dim; TMA
// load) and the batch as N (16..128; filled by the CTA's threads, because the activation
// side needs a dtype conversion or a merge on the way in). 512 threads: these kernels are
// short chains of dependent steps, so four warps per scheduler hide each other's latencies;
// in the epilogue warp w reads TMEM lane quadrant w % 4, column group w / 4.
#pragma once

#include "common.cuh"
#include "decode.cuh"

namespace mlra {

constexpr float kLog2e = 1.4426950408889634f;
// threads of the combine / up-projection kernel: 16 warps, so the latency-bound merge and the
// epilogue are spread over four warps per scheduler
constexpr int kProjThreads = 512;
constexpr float kLn2 = 0.6931471805599453f;

struct ProjParams {
  // absorb
  const void* q;      // [B][h][d_h + d_r]
  int q_f32;          // 1: fp32 q, 0: bf16 q
  __nv_bfloat16* q_pack;  // [B][nsub][NP][DB + DR]
  float qscale;       // softmax scale * log2(e)
  int d_r;
  int np;             // heads per decode CTA (rows per q_pack block)
  int nsub;           // decode CTAs per group
  int chunks;         // head chunks per latent block
  int heads_block;    // h / k
  // uproj
  const float* o_part;
  const float* lse_part;
  void* out;          // [B][h][d_h]
  int out_f32;
  float* lse_out;     // [B][h] natural log, nullable
  float* latent_out;  // [B][h][DB] fp32 (combine-only mode)
  const int* seq_lens;
  int pt_stride;
  int groups;
  // common
  int batch;
  int h;              // heads of the packed query and the partials (k*h virtual heads when the
                      // blocks are summed)
  int q_heads;        // heads of the query rows (head v reads query row v % q_heads)
  int out_heads;      // heads of the output rows
  float out_scale;    // alpha_attn when the blocks are summed, else 1
  // E4M3 cache (absorb writes each head's query as two E4M3 terms with a power-of-two factor)
  float latent_scale;  // value of a latent byte = latent_scale * e4m3(byte)
  float rope_scale;    // value of a RoPE byte = rope_scale * e4m3(byte)
  float* qfac;         // [B][nsub][np] factor of each head's query terms
  int q_rows_per_sub;  // query rows per (sequence, decode CTA): np, or 2 * np for two terms
  int* status;        // cleared by absorb CTA (0, 0); written by the combine kernel
  EarlyTags tags;     // absorb errors (the decode kernel folds them into status)
  unsigned long long wait_limit_ns;
  int inject_stall;   // test hook: 2 = absorb CTA (1, 0) never issues its MMA, so its wait runs out
};

template <int DB_, int DH_, int NT_>
struct ProjShape {
  static constexpr int DB = DB_, DH = DH_, NT = NT_;
  // absorb: A = W^UK_h [DB rows][DH cols], K-major, K split into swizzle-width regions
  static constexpr int AW = DH < 64 ? DH : 64;
  static constexpr int NKR = DH / AW;
  static constexpr int AROWB = AW * 2;
  static constexpr int NMT = DB >= 128 ? DB / 128 : 1;
  static constexpr int A1_REG = round_up(NMT * 128 * AROWB, 1024);
  static constexpr int B1_REG = round_up(NT * AROWB, 1024);
  static constexpr int A1_BOXR = NMT * 128 < 256 ? NMT * 128 : 256;
  static constexpr int A1_TX = NKR * NMT * 128 * AROWB;
  // q^R rows of the batch tile (bf16 query: loaded by TMA, then scaled into the packed query);
  // room for d_rope up to 64
  static constexpr int OFF_QRS = NKR * A1_REG + NKR * B1_REG;
  static constexpr int QRS_BYTES = round_up(NT * 64 * 2, 1024);
  // operand tiles, reused afterwards to stage the output rows
  static constexpr int STG1 = round_up(OFF_QRS + QRS_BYTES > NT * DB * 2 ? OFF_QRS + QRS_BYTES : NT * DB * 2, 1024);
  static constexpr int SMEM1 = STG1 + 1024 + 256;
  // E4M3 output: the fp32 query rows [NT][DB + up to 64 RoPE columns] are staged after the
  // barriers, then each is split into two E4M3 terms
  static constexpr int OFF_STF = STG1 + 256;
  static constexpr int SMEM1F8 = OFF_STF + NT * (DB + 64) * 4 + 1024;
  static constexpr int TMEM1 = NMT * NT <= 32 ? 32 : NMT * NT <= 64 ? 64 : NMT * NT <= 128 ? 128 :
                               NMT * NT <= 256 ? 256 : 512;
  // uproj: A = (W^UV_h)^T, MN-major: atoms of AW output columns, each DB rows (K) deep
  static constexpr int ATOM = round_up(DB * AROWB, 1024);
  static constexpr int NATOM = DH / AW;  // real atoms; M = 128 repeats the last via LBO = 0
  static constexpr uint32_t A4_LBO = DH >= 128 ? ATOM : 0;
  static constexpr int A4_BOXR = DB < 256 ? DB : 256;
  static constexpr int A4_TX = NATOM * DB * AROWB;
  static constexpr int BW = DB < 64 ? DB : 64;  // õ regions (K-major)
  static constexpr int NKB = DB / BW;
  static constexpr int BROWB = BW * 2;
  static constexpr int B4_REG = round_up(NT * BROWB, 1024);
  static constexpr int STG4 = round_up(NATOM * ATOM + NKB * B4_REG > NT * DH * 4 ? NATOM * ATOM + NKB * B4_REG
                                                                                  : NT * DH * 4, 1024);
  static constexpr int SMEM4 = STG4 + 1024 + 1024 + NT * 11 * 4;
  static constexpr int TMEM4 = NT <= 32 ? 32 : NT <= 64 ? 64 : 128;
  static_assert(DH <= 128, "one M tile of head dim");

};

// ---------------------------------------------------------------------------------------
// absorb
// ---------------------------------------------------------------------------------------
// F8: the packed query is written for an E4M3 cache: row [q~ * latent_scale | q^R * rope_scale]
// (times scale * log2 e) of each (sequence, head) is multiplied by a power of two 2^E that puts
// its largest magnitude in [128, 256), and stored as two E4M3 terms (hi: the nearest E4M3
// value, lo: the nearest to the remainder) in rows prow and np + prow; qfac receives 2^-E.
template <class Sh, bool F8 = false>
__global__ void __launch_bounds__(kProjThreads, 1)
    mlra_absorb_kernel(const __grid_constant__ CUtensorMap map_wuk, const __grid_constant__ CUtensorMap map_qc,
                       const __grid_constant__ CUtensorMap map_qr, const ProjParams p) {
  constexpr int DB = Sh::DB, DH = Sh::DH, NT = Sh::NT;
  static_assert(NT * DB * 2 <= Sh::OFF_QRS, "output staging must not overlap the q^R staging");
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  MLRA_TRACE_INIT
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* A = smem;
  uint8_t* Bq = smem + Sh::NKR * Sh::A1_REG;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sh::STG1);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  float* stf = reinterpret_cast<float*>(smem + Sh::OFF_STF);  // F8 only: [NT][DB + d_r] fp32

  const int head = blockIdx.x;
  const int n0 = blockIdx.y * NT;
  const int warp = warp_id(), lane = lane_id();
  const int qw = DB + p.d_r;
  bool mma_issued = false;  // (warp 0) the MMA went out: its commit is drained at teardown
  const int hb = head % p.heads_block;
  const int blk = head / p.heads_block;
  const int sub = blk * p.chunks + hb / p.np;
  const int prow = hb % p.np;

  if (threadIdx.x == 0) MLRA_TRACE_POINT(0, 0);
  // a bf16 query comes in by TMA with the weight: [batch tile][q^C columns] straight into the
  // MMA's swizzled B layout, [batch tile][q^R] into a staging tile (rows past the batch read 0)
  const bool tma_q = !p.q_f32;
  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort_flag = 0;
    fence_mbar_init();
    // issue the loads first: nothing below depends on them until the MMA. The weight does not
    // depend on the previous kernel in the stream, so it streams in while that kernel finishes
    // (programmatic dependent launch); the query, the status word and the packed-query output
    // wait for it.
    const uint64_t pol = l2_policy_evict_first();
    mbar_arrive_expect_tx(&bars[0], Sh::A1_TX + (tma_q ? NT * (DH + p.d_r) * 2 : 0));
    for (int kr = 0; kr < Sh::NKR; ++kr)
      for (int r0 = 0; r0 < Sh::NMT * 128; r0 += Sh::A1_BOXR)
        tma_load_2d(A + kr * Sh::A1_REG + r0 * Sh::AROWB, &map_wuk, &bars[0], kr * Sh::AW, head * DB + r0, pol);
    grid_dependency_wait();
    if (blockIdx.x == 0 && blockIdx.y == 0) clear_status_and_tags(p.status, p.tags);
    if (tma_q) {
      const int qh = head % p.q_heads;
      for (int kr = 0; kr < Sh::NKR; ++kr)
        tma_load_3d(Bq + kr * Sh::B1_REG, &map_qc, &bars[0], kr * Sh::AW, qh, n0, pol);
      tma_load_3d(smem + Sh::OFF_QRS, &map_qr, &bars[0], DH, qh, n0, pol);
    }
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, Sh::TMEM1);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  grid_dependency_wait();  // (returns at once: thread 0 has waited for the previous kernel)
  const uint32_t tbase = *tmem_slot;
  if (threadIdx.x == 0) MLRA_TRACE_POINT(0, 1);
  // let the decode kernel's CTAs start (on SMs this grid leaves free) and run their set-up and
  // split planning now; they wait for this grid's results before reading them
  grid_launch_dependents();

  // q_h for the batch tile, in 8-element chunks: q^C chunks -> bf16, K-major swizzled tile
  // (the MMA's B operand); q^R chunks -> packed query, scaled. All global loads of a round are
  // issued before any store, so the round costs one memory round trip.
  if (!tma_q) {
    const int qwh = DH + p.d_r;        // elements of one q row
    const int cpr = qwh / 8;           // chunks per row
    const int nch = NT * cpr;
    constexpr int RND = 2;
    if (threadIdx.x == 0) MLRA_TRACE_POINT(0, 10);
    for (int base = 0; base < nch; base += kProjThreads * RND) {
      float v[RND][8];
      bool use[RND];
#pragma unroll
      for (int i = 0; i < RND; ++i) {
        const int idx = base + i * kProjThreads + threadIdx.x;
        const int bl = idx / cpr, d8 = (idx % cpr) * 8;
        const int b = n0 + bl;
        use[i] = idx < nch;
        if (use[i] && b < p.batch) {
          const size_t off = ((size_t)b * p.q_heads + head % p.q_heads) * qwh + d8;
          if (p.q_f32) {
            const float4* src = reinterpret_cast<const float4*>(static_cast<const float*>(p.q) + off);
            const float4 x0 = __ldg(src), x1 = __ldg(src + 1);
            v[i][0] = x0.x; v[i][1] = x0.y; v[i][2] = x0.z; v[i][3] = x0.w;
            v[i][4] = x1.x; v[i][5] = x1.y; v[i][6] = x1.z; v[i][7] = x1.w;
          } else {
            const uint4 raw = __ldg(reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.q) + off));
            const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float2 f = __bfloat1622float2(h2[e]);
              v[i][2 * e] = f.x;
              v[i][2 * e + 1] = f.y;
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < 8; ++e) v[i][e] = 0.f;
        }
      }
#pragma unroll
      for (int i = 0; i < RND; ++i) {
        if (!use[i]) continue;
        const int idx = base + i * kProjThreads + threadIdx.x;
        const int bl = idx / cpr, d8 = (idx % cpr) * 8;
        if (d8 < DH) {
          uint4 w;
          w.x = pack_bf16x2(v[i][0], v[i][1]);
          w.y = pack_bf16x2(v[i][2], v[i][3]);
          w.z = pack_bf16x2(v[i][4], v[i][5]);
          w.w = pack_bf16x2(v[i][6], v[i][7]);
          *reinterpret_cast<uint4*>(Bq + (d8 / Sh::AW) * Sh::B1_REG +
                                    swizzle(bl * Sh::AROWB + (d8 % Sh::AW) * 2, Sh::AROWB)) = w;
        } else if (F8) {
#pragma unroll
          for (int e = 0; e < 8; ++e) stf[bl * qw + DB + (d8 - DH) + e] = v[i][e] * p.qscale * p.rope_scale;
        } else if (n0 + bl < p.batch) {
          uint4 w;
          w.x = pack_bf16x2(v[i][0] * p.qscale, v[i][1] * p.qscale);
          w.y = pack_bf16x2(v[i][2] * p.qscale, v[i][3] * p.qscale);
          w.z = pack_bf16x2(v[i][4] * p.qscale, v[i][5] * p.qscale);
          w.w = pack_bf16x2(v[i][6] * p.qscale, v[i][7] * p.qscale);
          *reinterpret_cast<uint4*>(p.q_pack + (((size_t)(n0 + bl) * p.nsub + sub) * p.np + prow) * qw + DB +
                                    (d8 - DH)) = w;
        }
      }
    }
  }
  if (threadIdx.x == 0) MLRA_TRACE_POINT(0, 11);
  // rows of a head chunk that no head fills (h/k below the MMA width) are never read: the
  // decode kernel loads only the real rows and keeps the rest zero in shared memory
  if (threadIdx.x == 0) MLRA_TRACE_POINT(0, 12);
  fence_proxy_async_smem();
  if (threadIdx.x == 0) MLRA_TRACE_POINT(0, 13);
  __syncthreads();
  if (threadIdx.x == 0) MLRA_TRACE_POINT(0, 2);

  const bool stall = p.inject_stall == 2 && blockIdx.x == 1 && blockIdx.y == 0;
  if (warp == 0) {
    const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[0], 0, abort_flag, p.wait_limit_ns));
    if (ok && !stall) {
      tc_fence_after();
      if (lane == 0) {
        MLRA_TRACE_POINT(0, 3);
        constexpr uint32_t idesc = idesc_bf16_f32(128, NT, false, false);
        constexpr int KPR = Sh::AW / 16;  // MMA K steps per region
#pragma unroll
        for (int mt = 0; mt < Sh::NMT; ++mt)
#pragma unroll
          for (int ks = 0; ks < DH / 16; ++ks) {
            const uint64_t a = smem_desc(smem_u32(A + (ks / KPR) * Sh::A1_REG + mt * 128 * Sh::AROWB +
                                                  (ks % KPR) * 32),
                                         16, 8 * Sh::AROWB, swizzle_code(Sh::AROWB));
            const uint64_t b = smem_desc(smem_u32(Bq + (ks / KPR) * Sh::B1_REG + (ks % KPR) * 32), 16,
                                         8 * Sh::AROWB, swizzle_code(Sh::AROWB));
            umma_bf16(tbase + mt * NT, a, b, idesc, ks > 0 ? 1u : 0u);
          }
        umma_commit(&bars[1]);
      }
      __syncwarp();
      mma_issued = true;
    }
  }
  if (tma_q && warp != 0) {
    // q^R from the staging tile, scaled, into the packed query (while warp 0 runs the MMA)
    if (mbar_wait(&bars[0], 0, abort_flag, p.wait_limit_ns)) {
      const int cpr = p.d_r / 8;
      const __nv_bfloat16* qrs = reinterpret_cast<const __nv_bfloat16*>(smem + Sh::OFF_QRS);
      for (int idx = threadIdx.x - 32; idx < NT * cpr; idx += kProjThreads - 32) {
        const int bl = idx / cpr, c8 = (idx % cpr) * 8;
        const int b = n0 + bl;
        if (b >= p.batch) continue;
        const uint4 raw = *reinterpret_cast<const uint4*>(qrs + bl * p.d_r + c8);
        const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&raw);
        float f[8];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 v = __bfloat1622float2(h2[e]);
          f[2 * e] = v.x * p.qscale;
          f[2 * e + 1] = v.y * p.qscale;
        }
        if constexpr (F8) {
#pragma unroll
          for (int e = 0; e < 8; ++e) stf[bl * qw + DB + c8 + e] = f[e] * p.rope_scale;
          continue;
        }
        uint4 w;
        w.x = pack_bf16x2(f[0], f[1]);
        w.y = pack_bf16x2(f[2], f[3]);
        w.z = pack_bf16x2(f[4], f[5]);
        w.w = pack_bf16x2(f[6], f[7]);
        *reinterpret_cast<uint4*>(p.q_pack + (((size_t)b * p.nsub + sub) * p.np + prow) * qw + DB + c8) = w;
      }
    }
  }
  const bool ok = mbar_wait(&bars[1], 0, abort_flag, p.wait_limit_ns);
  if (threadIdx.x == 0) MLRA_TRACE_POINT(0, 4);
  if (ok) {
    // D^T (lanes = latent features, columns = batch rows) -> bf16 rows [b][c] in shared
    // memory (the weight tile is no longer read), then 16-byte stores of whole rows. Warp w
    // reads lane quadrant w % 4 (the quadrant its warp id may access) and column group w / 4.
    constexpr int COLS = NT / 4 >= 8 ? NT / 4 : 8;
    const int q4 = warp & 3, cg = warp >> 2;
    if (cg * COLS < NT) {
      tc_fence_after();
      const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
      __nv_bfloat16* stage_out = reinterpret_cast<__nv_bfloat16*>(A);
#pragma unroll
      for (int mt = 0; mt < Sh::NMT; ++mt) {
        const int c = mt * 128 + q4 * 32 + lane;
        float v[COLS];
        tmem_load_row<COLS>(tbase + lane_base + mt * NT + cg * COLS, v);
        tmem_ld_wait();
        if (c < DB) {
          if constexpr (F8) {
#pragma unroll
            for (int n = 0; n < COLS; ++n) stf[(cg * COLS + n) * qw + c] = v[n] * p.qscale * p.latent_scale;
          } else {
#pragma unroll
            for (int n = 0; n < COLS; ++n)
              stage_out[(cg * COLS + n) * DB + c] = __float2bfloat16_rn(v[n] * p.qscale);
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (ok && !F8) {
    for (int idx = threadIdx.x; idx < NT * (DB / 8); idx += kProjThreads) {
      const int n = idx / (DB / 8), c8 = (idx % (DB / 8)) * 8;
      const int b = n0 + n;
      if (b < p.batch)
        *reinterpret_cast<uint4*>(p.q_pack + (((size_t)b * p.nsub + sub) * p.np + prow) * qw + c8) =
            *reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(A) + n * DB + c8);
    }
  }
  if (ok && F8) {
    // one warp per batch row: the row's largest magnitude fixes its power of two, then each
    // lane splits 8 consecutive elements into the two E4M3 terms
    uint8_t* qp8 = reinterpret_cast<uint8_t*>(p.q_pack);
    for (int n = warp; n < NT; n += kProjThreads / 32) {
      const int b = n0 + n;
      if (b >= p.batch) continue;
      const float* row = stf + n * qw;
      float amax = 0.f;
      for (int i = lane; i < qw; i += 32) amax = fmaxf(amax, fabsf(row[i]));
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      int ex = 0;
      if (amax > 0.f) frexpf(amax, &ex);          // amax in [2^(ex-1), 2^ex)
      const int e = amax > 0.f ? min(max(8 - ex, -120), 120) : 0;
      const float up = ldexpf(1.f, e);           // amax * up in [128, 256)
      const size_t hi_row = ((size_t)b * p.nsub + sub) * p.q_rows_per_sub + prow;
      const size_t lo_row = hi_row + p.np;
      for (int c8 = lane * 8; c8 < qw; c8 += 32 * 8) {
        uint32_t hw[2], lw[2];
#pragma unroll
        for (int e2 = 0; e2 < 4; ++e2) {
          const float x0 = row[c8 + 2 * e2] * up, x1 = row[c8 + 2 * e2 + 1] * up;
          const uint16_t h2 = e4m3x2_from_f32(x0, x1);
          const uint32_t hf = f16x2_from_e4m3x2(h2);
          const float2 hv = __half22float2(*reinterpret_cast<const __half2*>(&hf));
          const uint16_t l2 = e4m3x2_from_f32(x0 - hv.x, x1 - hv.y);
          if (e2 % 2 == 0) {
            hw[e2 / 2] = h2;
            lw[e2 / 2] = l2;
          } else {
            hw[e2 / 2] |= static_cast<uint32_t>(h2) << 16;
            lw[e2 / 2] |= static_cast<uint32_t>(l2) << 16;
          }
        }
        *reinterpret_cast<uint2*>(qp8 + hi_row * qw + c8) = make_uint2(hw[0], hw[1]);
        *reinterpret_cast<uint2*>(qp8 + lo_row * qw + c8) = make_uint2(lw[0], lw[1]);
      }
      if (lane == 0) p.qfac[((size_t)b * p.nsub + sub) * p.np + prow] = ldexpf(1.f, -e);
    }
  }
  // drain before releasing TMEM and shared memory
  if (threadIdx.x == 0) MLRA_TRACE_POINT(0, 5);
  bool drained = true;
  if (threadIdx.x == 0) {
    drained = mbar_wait_drain(&bars[0], 0, p.wait_limit_ns);
    if (mma_issued) drained = mbar_wait_drain(&bars[1], 0, p.wait_limit_ns) && drained;
  }
  tc_fence_before();
  __syncthreads();
  // this kernel may fail before CTA (0, 0) has cleared the status word: report by tag
  if (threadIdx.x == 0 && *abort_flag) report_early(p.tags, kTagTimeout);
  if (threadIdx.x == 0 && !drained) report_early(p.tags, kTagDrain);
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, Sh::TMEM1);
  }
}

// ---------------------------------------------------------------------------------------
// combine + uproj (LATENT_ONLY: combine and write o~ in fp32, no projection)
// ---------------------------------------------------------------------------------------
// SUMK > 1 (summed blocks): the CTA of output head `head` merges the partials of its SUMK
// virtual heads j*out_heads + head (latent block j), lays them side by side along K
// (DB = SUMK * block width) and multiplies by the SUMK stacked W^UV matrices in one GEMM, so
// the sum over blocks happens in the tensor core's accumulator; out_scale applies alpha_attn.
template <class Sh, bool LATENT_ONLY, int SUMK = 1>
__global__ void __launch_bounds__(kProjThreads, 1)
    mlra_uproj_kernel(const __grid_constant__ CUtensorMap map_wuv, const ProjParams p) {
  constexpr int DB = Sh::DB, DH = Sh::DH, NT = Sh::NT;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  MLRA_TRACE_INIT
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* A = smem;
  uint8_t* Bo = smem + Sh::NATOM * Sh::ATOM;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Sh::STG4);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* err_flag = const_cast<int*>(reinterpret_cast<volatile int*>(tmem_slot + 2));
  int* scratch = reinterpret_cast<int*>(tmem_slot + 4);  // 40 ints
  int* pref = scratch + 40;                              // NT ints

  const int head = blockIdx.x;
  const int n0 = blockIdx.y * NT;
  const int warp = warp_id(), lane = lane_id();
  const int cap_len = p.pt_stride * kPage;
  if (threadIdx.x == 0) MLRA_TRACE_POINT(2, 0);

  if (threadIdx.x == 0) {
    mbar_init(&bars[0], 1);
    mbar_init(&bars[1], 1);
    *abort_flag = 0;
    *err_flag = 0;
    fence_mbar_init();
  }
  if (!LATENT_ONLY && warp == 0) {
    tmem_alloc(tmem_slot, Sh::TMEM4);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = LATENT_ONLY ? 0u : *tmem_slot;

  // the weight does not depend on the previous kernel: load it before waiting for it
  if (!LATENT_ONLY && threadIdx.x == 0) {
    tma_prefetch_map(&map_wuv);
    mbar_arrive_expect_tx(&bars[0], Sh::A4_TX);
    const uint64_t pol = l2_policy_evict_first();
    constexpr int DBB = DB / SUMK;  // rows of one block's W^UV
    constexpr int BOXR = DBB < Sh::A4_BOXR ? DBB : Sh::A4_BOXR;
    for (int a = 0; a < Sh::NATOM; ++a)
      for (int j = 0; j < SUMK; ++j)
        for (int r0 = 0; r0 < DBB; r0 += BOXR)
          tma_load_2d(A + a * Sh::ATOM + (j * DBB + r0) * Sh::AROWB, &map_wuv, &bars[0], a * Sh::AW,
                      (j * p.out_heads + head) * DBB + r0, pol);
  }

  // plan: total tiles, and where each sequence of this batch tile starts in the flattened
  // tile order. Small batches: every warp computes it alone (no block barrier); large ones:
  // a block-wide scan into pref[].
  int err = 0;
  WarpPlan wp;
  const bool warp_plan = warp_plan_load(p.seq_lens, p.batch, cap_len, wp, &err);
  int T;
  if (warp_plan) {
    T = wp.total;
  } else {
    T = block_total_tiles(p.seq_lens, p.batch, cap_len, scratch, &err);
    int running = 0;
    for (int base = 0; base < min(p.batch, n0 + NT); base += blockDim.x) {
      const int b = base + threadIdx.x;
      const int t = b < p.batch ? tiles_of(clamp_len(__ldg(p.seq_lens + b), cap_len, &err)) : 0;
      int chunk_total;
      const int pb = running + block_scan_tiles(t, scratch, &chunk_total);
      if (b >= n0 && b < n0 + NT) pref[b - n0] = pb;
      running += chunk_total;
    }
    __syncthreads();
  }
  const int quota = T > 0 ? (T + p.groups - 1) / p.groups : 1;
  if (err) atomicOr(err_flag, 1);
  if (threadIdx.x == 0) MLRA_TRACE_POINT(2, 1);

  grid_dependency_wait();  // the partials come from the decode kernel
  // the next kernel in the stream (the next step's absorb) may start its set-up and weight
  // loads now; it waits for this grid before touching anything this grid reads or writes
  grid_launch_dependents();
  if (threadIdx.x == 0) MLRA_TRACE_POINT(2, 2);

  // merge the split partials of each (sequence, head) and stage o~ as bf16 (K-major).
  // Warp w takes batch rows w*RB .. w*RB+RB-1 (then + NW*RB ...) and issues every load of a
  // round (the rows' lse values and partial vectors, up to SB segments each) before using
  // any of them, so a round costs one memory round trip.
  constexpr int NW = kProjThreads / 32;
  constexpr int PER = DB / 32;  // features per lane
  constexpr int DBB = DB / SUMK;  // features of one block
  static_assert(DBB % PER == 0, "a lane's features lie in one block");
  // the (virtual) head whose partials this lane merges, and the lane's first feature in it
  const int vhead = SUMK == 1 ? head : ((lane * PER) / DBB) * p.out_heads + head;
  const int f0 = (lane * PER) % DBB;
  constexpr int RB = PER >= 16 ? 1 : 2;  // rows per warp per round
  constexpr int SB = PER >= 8 ? 2 : 4;  // segments per row loaded together
  for (int r0 = warp * RB; r0 < NT; r0 += NW * RB) {
    int c0[RB], nsg[RB];
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) {
      const int bl = r0 + rb, b = n0 + bl;
      c0[rb] = 0;
      nsg[rb] = 0;
      if (bl < NT && b < p.batch) {
        int tb, pb;
        if (warp_plan) {
          pb = warp_plan_start(wp, b, &tb);
        } else {
          tb = tiles_of(clamp_len(__ldg(p.seq_lens + b), cap_len, &err));
          pb = pref[bl];
        }
        if (tb > 0) {
          c0[rb] = pb / quota;
          nsg[rb] = (pb + tb - 1) / quota - c0[rb] + 1;
        }
      }
    }
    float acc[RB][PER];
    float mx[RB], sum[RB];
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) {
      mx[rb] = -INFINITY;
      sum[rb] = 0.f;
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[rb][e] = 0.f;
    }
    int maxseg = 0;
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) maxseg = max(maxseg, nsg[rb]);
    if (threadIdx.x == 0) MLRA_TRACE_POINT(2, 7);
    for (int s0 = 0; s0 < maxseg; s0 += SB) {
      float lv[RB][SB];
      float v[RB][SB][PER];
#pragma unroll
      for (int rb = 0; rb < RB; ++rb) {
        const int b = n0 + r0 + rb;
#pragma unroll
        for (int si = 0; si < SB; ++si) {
          if (s0 + si < nsg[rb]) {
            const size_t slot = (size_t)(b + c0[rb] + s0 + si);
            lv[rb][si] = __ldg(p.lse_part + slot * p.h + vhead);
            const float* src = p.o_part + (slot * p.h + vhead) * DBB + f0;
            if constexpr (PER % 4 == 0) {
#pragma unroll
              for (int e = 0; e < PER; e += 4) {
                const float4 f = __ldg(reinterpret_cast<const float4*>(src + e));
                v[rb][si][e] = f.x; v[rb][si][e + 1] = f.y; v[rb][si][e + 2] = f.z; v[rb][si][e + 3] = f.w;
              }
            } else {
#pragma unroll
              for (int e = 0; e < PER; ++e) v[rb][si][e] = __ldg(src + e);
            }
          } else {
            lv[rb][si] = -INFINITY;
#pragma unroll
            for (int e = 0; e < PER; ++e) v[rb][si][e] = 0.f;
          }
        }
      }
      // online log-sum-exp merge (base 2) of this round's segments
#pragma unroll
      for (int rb = 0; rb < RB; ++rb) {
        float m_new = mx[rb];
#pragma unroll
        for (int si = 0; si < SB; ++si) m_new = fmaxf(m_new, lv[rb][si]);
        if (m_new == -INFINITY) continue;
        // ex2.approx: these weights lie in [0, 1] and the merge is fp32 (relative error ~2^-22)
        const float sc = fast_exp2(mx[rb] - m_new);  // 0 when mx was -inf
        sum[rb] *= sc;
#pragma unroll
        for (int e = 0; e < PER; ++e) acc[rb][e] *= sc;
#pragma unroll
        for (int si = 0; si < SB; ++si) {
          const float wgt = fast_exp2(lv[rb][si] - m_new);  // 0 for absent segments
          sum[rb] += wgt;
#pragma unroll
          for (int e = 0; e < PER; ++e) acc[rb][e] += wgt * v[rb][si][e];
        }
        mx[rb] = m_new;
      }
    }
    if (threadIdx.x == 0) MLRA_TRACE_POINT(2, 8);
#pragma unroll
    for (int rb = 0; rb < RB; ++rb) {
      const int bl = r0 + rb, b = n0 + bl;
      if (bl >= NT) continue;
      // sum >= 1 (the largest segment's own weight is 1): div.approx is within 2 ulp
      const float inv = sum[rb] > 0.f ? __fdividef(1.f, sum[rb]) : 0.f;
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[rb][e] *= inv;
      if (b < p.batch && f0 == 0 && p.lse_out)  // one lane per (virtual) head
        p.lse_out[(size_t)b * p.h + vhead] = nsg[rb] > 0 ? (mx[rb] + __log2f(sum[rb])) * kLn2 : -INFINITY;
      if constexpr (LATENT_ONLY) {
        if (b < p.batch) {
          float* dst = p.latent_out + ((size_t)b * p.h + head) * DB + lane * PER;
#pragma unroll
          for (int e = 0; e < PER; ++e) dst[e] = acc[rb][e];
        }
      } else {
        // lane's PER features start at byte lane*PER*2 of the row
#pragma unroll
        for (int e = 0; e < PER; e += 2) {
          const int f = lane * PER + e;
          uint8_t* reg = Bo + (f / Sh::BW) * Sh::B4_REG;
          const uint32_t off = swizzle(bl * Sh::BROWB + (f % Sh::BW) * 2, Sh::BROWB);
          if constexpr (PER == 1) {
            *reinterpret_cast<__nv_bfloat16*>(reg + off) = __float2bfloat16_rn(acc[rb][0]);
          } else {
            *reinterpret_cast<uint32_t*>(reg + off) = pack_bf16x2(acc[rb][e], acc[rb][e + 1]);
          }
        }
      }
    }
    if (threadIdx.x == 0) MLRA_TRACE_POINT(2, 9);
  }
  if (threadIdx.x == 0) MLRA_TRACE_POINT(2, 3);
  if (err) atomicOr(err_flag, 1);

  bool mma_issued = false;  // (warp 0) the MMA went out: its commit is drained at teardown
  if constexpr (!LATENT_ONLY) {
    fence_proxy_async_smem();
    __syncthreads();
    if (threadIdx.x == 0) MLRA_TRACE_POINT(2, 4);
    if (warp == 0) {
      const bool ok = __all_sync(0xffffffffu, mbar_wait(&bars[0], 0, abort_flag, p.wait_limit_ns));
      if (ok) {
        tc_fence_after();
        if (lane == 0) {
          constexpr uint32_t idesc = idesc_bf16_f32(128, NT, true, false);
          constexpr int KPR = Sh::BW / 16;
#pragma unroll
          for (int ks = 0; ks < DB / 16; ++ks) {
            const uint64_t a = smem_desc(smem_u32(A + ks * 16 * Sh::AROWB), Sh::A4_LBO, 8 * Sh::AROWB,
                                         swizzle_code(Sh::AROWB));
            const uint64_t b = smem_desc(smem_u32(Bo + (ks / KPR) * Sh::B4_REG + (ks % KPR) * 32), 16,
                                         8 * Sh::BROWB, swizzle_code(Sh::BROWB));
            umma_bf16(tbase, a, b, idesc, ks > 0 ? 1u : 0u);
          }
          umma_commit(&bars[1]);
        }
        __syncwarp();
        mma_issued = true;
      }
    }
    const bool ok = mbar_wait(&bars[1], 0, abort_flag, p.wait_limit_ns);
    if (threadIdx.x == 0) MLRA_TRACE_POINT(2, 5);
    if (ok) {
      // D^T (lanes = head-dim d, columns = batch rows) -> rows [b][d] in shared memory (the
      // operand tiles are no longer read), then 16-byte stores of whole output rows. Warp w
      // reads lane quadrant w % 4 (the quadrant its warp id may access) and column group w / 4.
      constexpr int COLS = NT / 4 >= 8 ? NT / 4 : 8;
      const int q4 = warp & 3, cg = warp >> 2;
      const int d = q4 * 32 + lane;
      if (cg * COLS < NT) {
        tc_fence_after();
        float v[COLS];
        tmem_load_row<COLS>(tbase + (static_cast<uint32_t>(q4 * 32) << 16) + cg * COLS, v);
        tmem_ld_wait();
        if (d < DH) {
          if (p.out_f32) {
            float* so = reinterpret_cast<float*>(A);
#pragma unroll
            for (int c = 0; c < COLS; ++c) so[(cg * COLS + c) * DH + d] = v[c] * p.out_scale;
          } else {
            __nv_bfloat16* so = reinterpret_cast<__nv_bfloat16*>(A);
#pragma unroll
            for (int c = 0; c < COLS; ++c) so[(cg * COLS + c) * DH + d] = __float2bfloat16_rn(v[c] * p.out_scale);
          }
        }
      }
    }
    tc_fence_before();
    __syncthreads();
    if (ok) {
      const int esz = p.out_f32 ? 4 : 2;
      const int chunks = DH * esz / 16;  // 16-byte pieces per output row
      for (int idx = threadIdx.x; idx < NT * chunks; idx += kProjThreads) {
        const int n = idx / chunks, c = idx % chunks;
        const int b = n0 + n;
        if (b < p.batch)
          *reinterpret_cast<uint4*>(static_cast<char*>(p.out) + (((size_t)b * p.out_heads + head) * DH) * esz + c * 16) =
              *reinterpret_cast<const uint4*>(A + (size_t)n * DH * esz + c * 16);
      }
    }
    if (threadIdx.x == 0) MLRA_TRACE_POINT(2, 6);
    if (threadIdx.x == 0) {
      if (!mbar_wait_drain(&bars[0], 0, p.wait_limit_ns)) atomicOr(err_flag, 2);
      if (mma_issued && !mbar_wait_drain(&bars[1], 0, p.wait_limit_ns)) atomicOr(err_flag, 2);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    if (*err_flag & 1) set_status(p.status, kErrSeqLen);
    if (*abort_flag) set_status(p.status, kErrTimeout);
    if (*err_flag & 2) force_status(p.status, kErrDrain);
  }
  if (!LATENT_ONLY && warp == 0) {
    tc_fence_after();
    tmem_dealloc(tbase, Sh::TMEM4);
  }
}

}  // namespace mlra
