// decode_attention.cuh -- one new query token per sequence against the KV cache
// ("Build your own Llama 3 from scratch" §3.3 KV Cache and 六 inference: the
// step's single query attends to every cached position 0..start_pos).
//
// Memory-bound: every cached K and V row is read exactly once per step.  A CTA
// owns (sequence b, KV head g, key range) and serves all n_rep query heads of
// group g from the same K/V rows (GQA, §3.4: head h reads KV head h / n_rep),
// so repeat_kv is never formed.  Key ranges ("splits") spread one sequence
// over many SMs; a second kernel merges the per-split softmax partials.
#pragma once
#include "common.cuh"

namespace l3 {

// Partial record per (b, h, split): m (running max of the scaled scores),
// l (sum of exp(s - m)), acc[hd] (sum of exp(s - m) * v).  Stored as floats
// [B][H][splits][hd + 2].
template <int HD, int NREP>
__global__ void __launch_bounds__(128)
    decode_attention_split_kernel(const bf16* __restrict__ q, const bf16* __restrict__ k_cache,
                                  const bf16* __restrict__ v_cache, float* __restrict__ part,
                                  int H, int KV, int cap, int n_keys, int keys_per_split,
                                  int splits, float scale_log2) {
  constexpr int DPL = HD / 32;  // output dims per lane
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int j0 = split * keys_per_split;
  const int j1 = min(j0 + keys_per_split, n_keys);

  __shared__ __align__(16) float qs[NREP][HD];
  __shared__ float red_m[4][NREP], red_l[4][NREP];
  __shared__ float red_acc[4][NREP][HD];

  for (int i = threadIdx.x; i < NREP * HD; i += 128) {
    const int h = i / HD, d = i % HD;
    qs[h][d] = __bfloat162float(q[((size_t)b * H + g * NREP + h) * HD + d]) * scale_log2;
  }
  __syncthreads();

  float m[NREP], l[NREP], acc[NREP][DPL];
#pragma unroll
  for (int h = 0; h < NREP; ++h) {
    m[h] = -INFINITY;
    l[h] = 0.f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) acc[h][i] = 0.f;
  }

  const size_t row_stride = (size_t)KV * HD;  // elements between consecutive positions
  const bf16* kbase = k_cache + ((size_t)b * cap * KV + g) * HD;
  const bf16* vbase = v_cache + ((size_t)b * cap * KV + g) * HD;

  for (int c0 = j0 + warp * 32; c0 < j1; c0 += 128) {
    // scores of key c0 + lane for every head (log2 domain)
    const int j = c0 + lane;
    float s[NREP];
#pragma unroll
    for (int h = 0; h < NREP; ++h) s[h] = 0.f;
    if (j < j1) {
      const uint4* kr = reinterpret_cast<const uint4*>(kbase + (size_t)j * row_stride);
#pragma unroll 4
      for (int d8 = 0; d8 < HD / 8; ++d8) {
        const uint4 kk = __ldg(kr + d8);
        const float k0 = bf16lo(kk.x), k1 = bf16hi(kk.x), k2 = bf16lo(kk.y), k3 = bf16hi(kk.y);
        const float k4 = bf16lo(kk.z), k5 = bf16hi(kk.z), k6 = bf16lo(kk.w), k7 = bf16hi(kk.w);
#pragma unroll
        for (int h = 0; h < NREP; ++h) {
          const float4 qa = *reinterpret_cast<const float4*>(&qs[h][d8 * 8]);
          const float4 qb = *reinterpret_cast<const float4*>(&qs[h][d8 * 8 + 4]);
          s[h] = fmaf(qa.x, k0, fmaf(qa.y, k1, fmaf(qa.z, k2, fmaf(qa.w, k3, s[h]))));
          s[h] = fmaf(qb.x, k4, fmaf(qb.y, k5, fmaf(qb.z, k6, fmaf(qb.w, k7, s[h]))));
        }
      }
    }
    const int nvalid = min(32, j1 - c0);
    float p[NREP];
#pragma unroll
    for (int h = 0; h < NREP; ++h) {
      const float sv = lane < nvalid ? s[h] : -INFINITY;
      const float cmax = warp_max(sv);
      const float mn = fmaxf(m[h], cmax);
      const float corr = exp2f(m[h] - mn);
      p[h] = lane < nvalid ? exp2f(sv - mn) : 0.f;
      l[h] = l[h] * corr + warp_sum(p[h]);
#pragma unroll
      for (int i = 0; i < DPL; ++i) acc[h][i] *= corr;
      m[h] = mn;
    }
    // P.V: lane owns dims lane*DPL .. lane*DPL+DPL-1
    for (int jj = 0; jj < nvalid; ++jj) {
      const bf16* vr = vbase + (size_t)(c0 + jj) * row_stride + lane * DPL;
      float vv[DPL];
      if constexpr (DPL == 4) {
        const uint2 u = __ldg(reinterpret_cast<const uint2*>(vr));
        vv[0] = bf16lo(u.x); vv[1] = bf16hi(u.x); vv[2] = bf16lo(u.y); vv[3] = bf16hi(u.y);
      } else if constexpr (DPL == 2) {
        const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(vr));
        vv[0] = bf16lo(u); vv[1] = bf16hi(u);
      } else {
#pragma unroll
        for (int i = 0; i < DPL; ++i) vv[i] = __bfloat162float(vr[i]);
      }
#pragma unroll
      for (int h = 0; h < NREP; ++h) {
        const float ph = __shfl_sync(0xffffffffu, p[h], jj);
#pragma unroll
        for (int i = 0; i < DPL; ++i) acc[h][i] = fmaf(ph, vv[i], acc[h][i]);
      }
    }
  }

  // merge the four warps
#pragma unroll
  for (int h = 0; h < NREP; ++h) {
    if (lane == 0) { red_m[warp][h] = m[h]; red_l[warp][h] = l[h]; }
#pragma unroll
    for (int i = 0; i < DPL; ++i) red_acc[warp][h][lane * DPL + i] = acc[h][i];
  }
  __syncthreads();
  for (int i = threadIdx.x; i < NREP * (HD + 2); i += 128) {
    const int h = i / (HD + 2), c = i % (HD + 2);
    float mx = -INFINITY;
#pragma unroll
    for (int w = 0; w < 4; ++w) mx = fmaxf(mx, red_m[w][h]);
    float val = 0.f;
    if (c == 0) {
      val = mx;
    } else {
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        const float f = red_m[w][h] == -INFINITY ? 0.f : exp2f(red_m[w][h] - mx);
        val += f * (c == 1 ? red_l[w][h] : red_acc[w][h][c - 2]);
      }
    }
    part[(((size_t)b * H + g * NREP + h) * splits + split) * (HD + 2) + c] = val;
  }
}

// out[b, h, :] = sum_s e^(m_s - M) acc_s / sum_s e^(m_s - M) l_s
template <int HD>
__global__ void decode_attention_combine_kernel(const float* __restrict__ part, bf16* __restrict__ out,
                                                int splits) {
  const int bh = blockIdx.x;  // b * H + h
  const float* p = part + (size_t)bh * splits * (HD + 2);
  float mx = -INFINITY;
  for (int s = 0; s < splits; ++s) mx = fmaxf(mx, p[s * (HD + 2)]);
  for (int d = threadIdx.x; d < HD; d += blockDim.x) {
    float num = 0.f, den = 0.f;
    for (int s = 0; s < splits; ++s) {
      const float ms = p[s * (HD + 2)];
      const float f = ms == -INFINITY ? 0.f : exp2f(ms - mx);
      den += f * p[s * (HD + 2) + 1];
      num += f * p[s * (HD + 2) + 2 + d];
    }
    out[(size_t)bh * HD + d] = __float2bfloat16_rn(num / den);
  }
}

}  // namespace l3
