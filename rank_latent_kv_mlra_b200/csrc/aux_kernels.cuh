// aux_kernels.cuh - cache append (the write side of the paged latent cache) and a dump of
// the device split plan for tests.
#pragma once

#include "common.cuh"

namespace mlra {

// One warp per new token: row [c | k^R] goes to slot pos % 64 of page table entry pos / 64.
// fp32 input is rounded to bf16 to nearest-even.
__global__ void mlra_append_kernel(__nv_bfloat16* __restrict__ pool, int num_pages,
                                   const int* __restrict__ page_table, int pt_stride, int batch,
                                   const int* __restrict__ seq_ids, const int* __restrict__ positions,
                                   const void* c_new, const void* kr_new, int in_f32, int n_tokens,
                                   int d_c, int d_r, int* status) {
  const int i = blockIdx.x * (blockDim.x / 32) + warp_id();
  const int lane = lane_id();
  if (i >= n_tokens) return;
  const int b = __ldg(seq_ids + i), pos = __ldg(positions + i);
  if (b < 0 || b >= batch || pos < 0 || pos / kPage >= pt_stride) {
    if (lane == 0) set_status(status, kErrSeqLen);
    return;
  }
  const int page = __ldg(page_table + (size_t)b * pt_stride + pos / kPage);
  if (page < 0 || page >= num_pages) {
    if (lane == 0) set_status(status, kErrPageOob);
    return;
  }
  const int D = d_c + d_r;
  __nv_bfloat16* row = pool + ((size_t)page * kPage + pos % kPage) * D;
  for (int e = lane; e < D; e += 32) {
    float v;
    if (e < d_c) {
      const size_t s = (size_t)i * d_c + e;
      v = in_f32 ? __ldg(static_cast<const float*>(c_new) + s)
                 : __bfloat162float(__ldg(static_cast<const __nv_bfloat16*>(c_new) + s));
    } else {
      const size_t s = (size_t)i * d_r + (e - d_c);
      v = in_f32 ? __ldg(static_cast<const float*>(kr_new) + s)
                 : __bfloat162float(__ldg(static_cast<const __nv_bfloat16*>(kr_new) + s));
    }
    row[e] = __float2bfloat16_rn(v);
  }
}

// E4M3 cache: one warp per new token writes the bytes e4m3(v / scale) of its row (v / scale in
// fp32, then rounded to the nearest E4M3 value, ties to even, saturated at +-448); the latent
// columns use latent_scale, the RoPE columns rope_scale.
__global__ void mlra_append_e4m3_kernel(uint8_t* __restrict__ pool, int num_pages,
                                        const int* __restrict__ page_table, int pt_stride, int batch,
                                        const int* __restrict__ seq_ids, const int* __restrict__ positions,
                                        const void* c_new, const void* kr_new, int in_f32, int n_tokens,
                                        int d_c, int d_r, float latent_scale, float rope_scale, int* status) {
  const int i = blockIdx.x * (blockDim.x / 32) + warp_id();
  const int lane = lane_id();
  if (i >= n_tokens) return;
  const int b = __ldg(seq_ids + i), pos = __ldg(positions + i);
  if (b < 0 || b >= batch || pos < 0 || pos / kPage >= pt_stride) {
    if (lane == 0) set_status(status, kErrSeqLen);
    return;
  }
  const int page = __ldg(page_table + (size_t)b * pt_stride + pos / kPage);
  if (page < 0 || page >= num_pages) {
    if (lane == 0) set_status(status, kErrPageOob);
    return;
  }
  const int D = d_c + d_r;
  uint8_t* row = pool + ((size_t)page * kPage + pos % kPage) * D;
  for (int e = lane; e < D; e += 32) {
    float v;
    if (e < d_c) {
      const size_t s = (size_t)i * d_c + e;
      v = in_f32 ? __ldg(static_cast<const float*>(c_new) + s)
                 : __bfloat162float(__ldg(static_cast<const __nv_bfloat16*>(c_new) + s));
      v = __fdiv_rn(v, latent_scale);
    } else {
      const size_t s = (size_t)i * d_r + (e - d_c);
      v = in_f32 ? __ldg(static_cast<const float*>(kr_new) + s)
                 : __bfloat162float(__ldg(static_cast<const __nv_bfloat16*>(kr_new) + s));
      v = __fdiv_rn(v, rope_scale);
    }
    row[e] = static_cast<uint8_t>(e4m3x2_from_f32(v, 0.f) & 0xFF);
  }
}

// Single CTA: writes every segment (b, group, tile_begin, tile_end, slot) of the plan in
// group order, using the same device routines as the decode and combine kernels.
__global__ void __launch_bounds__(192, 1)
    mlra_plan_kernel(const int* __restrict__ seq_lens, int batch, int pt_stride, int groups,
                     int* __restrict__ out, int max_segments, int* __restrict__ count, int* status) {
  __shared__ Segment list[64];
  __shared__ int scratch[40];
  __shared__ int words[3];
  int err = 0;
  const int cap_len = pt_stride * kPage;
  // the decode kernel's planning: warp scan for small batches, block scans otherwise
  WarpPlan wp;
  const bool warp_plan = warp_plan_load(seq_lens, batch, cap_len, wp, &err);
  const int T = warp_plan ? wp.total : block_total_tiles(seq_lens, batch, cap_len, scratch, &err);
  const int quota = T > 0 ? (T + groups - 1) / groups : 1;
  int written = 0;
  for (int g = 0; g < groups; ++g) {
    const int lo = min(g * quota, T), hi = min(lo + quota, T);
    if (lo >= hi) break;
    int b_start = 0, p_start = 0, more = 1;
    bool first = true;
    while (more) {
      int rb = batch, rp = 0, n;
      if (first && warp_plan) {
        if (threadIdx.x < 32) {
          const int total = warp_plan_segments(wp, lo, hi, list, 64, &rb, &rp);
          if (threadIdx.x == 0) {
            words[0] = total;
            words[1] = rb;
            words[2] = rp;
          }
        }
        __syncthreads();
        n = min(words[0], 64);
        more = words[0] > 64;
        rb = words[1];
        rp = words[2];
      } else {
        n = block_collect_segments(seq_lens, batch, cap_len, lo, hi, b_start, p_start, list, 64, scratch, &more,
                                   &rb, &rp, &err);
      }
      first = false;
      if (threadIdx.x == 0) {
        for (int i = 0; i < n; ++i, ++written) {
          if (written >= max_segments) continue;
          int* o = out + 5 * written;
          o[0] = list[i].b;
          o[1] = g;
          o[2] = list[i].tile_begin;
          o[3] = list[i].tile_end;
          o[4] = list[i].b + g;
        }
      }
      __syncthreads();
      b_start = rb;
      p_start = rp;
    }
  }
  if (threadIdx.x == 0) {
    *count = written;
    if (err) set_status(status, kErrSeqLen);
  }
}

}  // namespace mlra
