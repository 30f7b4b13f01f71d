// simt.cuh -- plain CUDA-core kernels for every step of the decoder.
//
// They serve the fp32 models (tiny configs where tensor cores would not meet
// a 1e-4 tolerance) and act as the independent GPU-side cross-check of the
// tcgen05 kernels.  Templated on the element type T (float or bf16); all
// arithmetic is fp32.  Nothing here is tuned.
#pragma once
#include "common.cuh"

namespace l3 {

// ---- embedding gather ("从0开发大模型—译llama3-from-scratch" §4) -------------
template <typename T>
__global__ void embed_kernel(const int32_t* __restrict__ ids, const T* __restrict__ table,
                             T* __restrict__ x, int D, int vocab) {
  griddep_wait_and_release();
  const int t = blockIdx.x;
  const int id = ids[t];
  const bool ok = id >= 0 && id < vocab;
  if (!ok && threadIdx.x == 0) record_error(LLAMA3_ERR_TOKEN);
  const T* src = table + (size_t)(ok ? id : 0) * D;
  T* dst = x + (size_t)t * D;
  if ((D * sizeof(T)) % 16 == 0) {   // rows are 16-byte aligned: copy 16 bytes per thread
    const int n16 = D * (int)sizeof(T) / 16;
    const uint4* s4 = reinterpret_cast<const uint4*>(src);
    uint4* d4 = reinterpret_cast<uint4*>(dst);
    for (int i = threadIdx.x; i < n16; i += blockDim.x) d4[i] = ok ? s4[i] : make_uint4(0, 0, 0, 0);
  } else {
    for (int i = threadIdx.x; i < D; i += blockDim.x) dst[i] = ok ? src[i] : from_f<T>(0.f);
  }
}

// ---- row gather: out[r] = x[idx[r]] (rows of D elements, 16-byte chunks) -----
// An index outside [0, n_rows) is reported and its output row zeroed.
__global__ void gather_rows_kernel(const uint4* __restrict__ x, long long row_stride16, const int32_t* __restrict__ idx,
                                   int n_rows, uint4* __restrict__ out, int row16) {
  griddep_wait_and_release();
  const int r = blockIdx.x;
  const int i = idx[r];
  const bool ok = i >= 0 && i < n_rows;
  if (!ok && threadIdx.x == 0) record_error(LLAMA3_ERR_ARG);
  const uint4* src = x + (size_t)(ok ? i : 0) * row_stride16;
  for (int c = threadIdx.x; c < row16; c += blockDim.x) out[(size_t)r * row16 + c] = ok ? src[c] : make_uint4(0, 0, 0, 0);
}

// ---- generation bookkeeping ("Build your own Llama 3 from scratch" 六) -------
// After a step has written the next token of every sequence into ids:
// history[step][b] = ids[b] (while step < rows), positions[b] += 1, step += 1.
// With done (eos_id >= 0): a sequence whose done flag is set has its token
// replaced by eos_id (the page stops a sequence at its end token), a sequence
// emitting eos_id gets its flag set, and done[batch] = 1 once every sequence
// is done.  One CTA, so the step counter is read once and advanced after every
// write.
__global__ void generation_advance_kernel(int32_t* __restrict__ positions, int32_t* __restrict__ ids,
                                          int32_t* __restrict__ history, int32_t* __restrict__ step,
                                          int32_t* __restrict__ done, int eos_id, int batch, int rows,
                                          long long stride) {
  griddep_wait_and_release();
  __shared__ int t;
  if (threadIdx.x == 0) t = *step;
  __syncthreads();
  int all = 1;
  for (int b = threadIdx.x; b < batch; b += blockDim.x) {
    int id = ids[b];
    if (done) {
      // a sequence that has emitted the end token keeps emitting it
      if (done[b]) {
        id = eos_id;
        ids[b] = id;
      } else if (id == eos_id) {
        done[b] = 1;
      }
      all &= done[b] != 0;
    }
    if (t >= 0 && t < rows) history[(size_t)t * stride + b] = id;
    positions[b] += 1;
  }
  all = __syncthreads_and(all);
  if (threadIdx.x == 0) {
    *step = t + 1;
    if (done) done[batch] = all;
  }
}

// ---- RMSNorm ("Build your own Llama 3 from scratch" §3.1) -------------------
// One CTA per row; fp32 sum of squares, one rounding on output.
template <typename T>
__global__ void rmsnorm_kernel(const T* __restrict__ x, long long row_stride,
                               const T* __restrict__ w, T* __restrict__ y, int D, float eps) {
  griddep_wait_and_release();
  const T* xr = x + (size_t)blockIdx.x * row_stride;
  T* yr = y + (size_t)blockIdx.x * D;
  float ss = 0.f;
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    float v = to_f(xr[i]);
    ss = fmaf(v, v, ss);
  }
  __shared__ float red[32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  if (threadIdx.x < 32) {
    float v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.f;
    v = warp_sum(v);
    if (threadIdx.x == 0) red[0] = v;
  }
  __syncthreads();
  float r = rsqrtf(red[0] / (float)D + eps);
  for (int i = threadIdx.x; i < D; i += blockDim.x) yr[i] = from_f<T>(to_f(xr[i]) * r * to_f(w[i]));
}

// bf16 rows with D % 8 == 0 and D <= 8 * 32 * CPL: one warp per row, the row
// held in registers as 16-byte chunks (one read of x, one write of y).
template <int CPL>
__global__ void __launch_bounds__(128) rmsnorm_bf16_warp_kernel(const bf16* __restrict__ x, long long row_stride,
                                                               const bf16* __restrict__ w, bf16* __restrict__ y,
                                                               int rows, int D, float eps) {
  griddep_wait_and_release();
  const int row = blockIdx.x * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (row >= rows) return;
  const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)row * row_stride);
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  uint4* yr = reinterpret_cast<uint4*>(y + (size_t)row * D);
  const int nchunk = D >> 3;
  uint4 v[CPL];
  float ss = 0.f;
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    const int c = lane + 32 * j;
    if (c < nchunk) {
      v[j] = xr[c];
      const uint32_t u[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float a = bf16lo(u[q]), b = bf16hi(u[q]);
        ss = fmaf(a, a, fmaf(b, b, ss));
      }
    }
  }
  ss = warp_sum(ss);
  const float r = rsqrtf(ss / (float)D + eps);
#pragma unroll
  for (int j = 0; j < CPL; ++j) {
    const int c = lane + 32 * j;
    if (c < nchunk) {
      const uint4 wv = __ldg(wr + c);
      const uint32_t u[4] = {v[j].x, v[j].y, v[j].z, v[j].w};
      const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
        o[q] = pack_bf16x2(bf16lo(u[q]) * r * bf16lo(ww[q]), bf16hi(u[q]) * r * bf16hi(ww[q]));
      yr[c] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// bf16 rows, few of them (decode): one CTA per row, one 16-byte chunk per
// thread (D % 8 == 0, D <= 8192), the weight chunk fetched before the
// reduction so both loads are in flight together.
__global__ void __launch_bounds__(1024) rmsnorm_bf16_row_kernel(const bf16* __restrict__ x, long long row_stride,
                                                               const bf16* __restrict__ w, bf16* __restrict__ y,
                                                               int D, float eps) {
  griddep_wait_and_release();
  const int row = blockIdx.x, c = threadIdx.x, lane = c & 31;
  const int nchunk = D >> 3;
  uint4 v = make_uint4(0, 0, 0, 0), wv = make_uint4(0, 0, 0, 0);
  if (c < nchunk) {
    v = reinterpret_cast<const uint4*>(x + (size_t)row * row_stride)[c];
    wv = __ldg(reinterpret_cast<const uint4*>(w) + c);
  }
  const uint32_t u[4] = {v.x, v.y, v.z, v.w};
  float ss = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float a = bf16lo(u[q]), b = bf16hi(u[q]);
    ss = fmaf(a, a, fmaf(b, b, ss));
  }
  __shared__ float red[32];
  ss = warp_sum(ss);
  if (lane == 0) red[c >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
  const int nw = (blockDim.x + 31) >> 5;
  for (int i = 0; i < nw; ++i) tot += red[i];
  const float r = rsqrtf(tot / (float)D + eps);
  if (c < nchunk) {
    const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q)
      o[q] = pack_bf16x2(bf16lo(u[q]) * r * bf16lo(ww[q]), bf16hi(u[q]) * r * bf16hi(ww[q]));
    reinterpret_cast<uint4*>(y + (size_t)row * D)[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// ---- GEMM C[m, n] = sum_k A[m, k] * B[n, k]   (fp32 result) -----------------
// 64x64 tile, 256 threads, 4x4 outputs per thread, K staged 16 at a time.
template <typename T>
__global__ void __launch_bounds__(256) gemm_simt_kernel(const T* __restrict__ A, const T* __restrict__ B,
                                                        float* __restrict__ C, int M, int N, int K,
                                                        int ldc) {
  griddep_wait_and_release();
  __shared__ float As[16][64 + 1];
  __shared__ float Bs[16][64 + 1];
  int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 64 * 16; i += 256) {
      int r = i >> 4, c = i & 15;
      int gm = m0 + r, gn = n0 + r, gk = k0 + c;
      As[c][r] = (gm < M && gk < K) ? to_f(A[(size_t)gm * K + gk]) : 0.f;
      Bs[c][r] = (gn < N && gk < K) ? to_f(B[(size_t)gn * K + gk]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int gm = m0 + ty * 4 + i;
    if (gm >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      int gn = n0 + tx * 4 + j;
      if (gn < N) C[(size_t)gm * ldc + gn] = acc[i][j];
    }
  }
}

// ---- epilogues over fp32 partial sums P[split][m][n] ------------------------
// (used after the SIMT GEMM with splits = 1 and after split-K tensor-core GEMMs)
// Four consecutive elements per thread: every row length here is a multiple of 4.
__device__ __forceinline__ void load4(const float* p, float (&v)[4]) {
  const float4 x = *reinterpret_cast<const float4*>(p);
  v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
}
__device__ __forceinline__ void load4(const bf16* p, float (&v)[4]) {
  const uint2 x = *reinterpret_cast<const uint2*>(p);
  v[0] = bf16lo(x.x); v[1] = bf16hi(x.x); v[2] = bf16lo(x.y); v[3] = bf16hi(x.y);
}
__device__ __forceinline__ void store4(float* p, const float (&v)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(bf16* p, const float (&v)[4]) {
  *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
}
// v = sum over s of P[s * split_stride + idx .. +3], added in split order;
// loads are issued four splits at a time so their latencies overlap.
__device__ __forceinline__ void sum4_splits(const float* P, int splits, long long split_stride, long long idx,
                                            float (&v)[4]) {
  load4(P + idx, v);
  int i = 1;
  for (; i + 4 <= splits; i += 4) {
    float w[4][4];
#pragma unroll
    for (int u = 0; u < 4; ++u) load4(P + (size_t)(i + u) * split_stride + idx, w[u]);
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int q = 0; q < 4; ++q) v[q] += w[u][q];
  }
  for (; i < splits; ++i) {
    float w[4];
    load4(P + (size_t)i * split_stride + idx, w);
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] += w[q];
  }
}

// out[m, n] = (res ? res[m, n] : 0) + P[m, n]
template <typename T>
__global__ void epi_residual_kernel(const float* __restrict__ P, int splits, long long split_stride,
                                    int ldp, const T* res, T* out, int M, int N) {
  griddep_wait_and_release();
  const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i >= (long long)M * N) return;
  const int m = (int)(i / N), n = (int)(i % N);
  float v[4];
  sum4_splits(P, splits, split_stride, (long long)m * ldp + n, v);
  if (res) {
    float r[4];
    load4(res + i, r);
#pragma unroll
    for (int q = 0; q < 4; ++q) v[q] += r[q];
  }
  store4(out + i, v);
}

// Residual add fused with the RMSNorm that follows it (decode, few rows):
//   x[m] <- round(x[m] + sum_s P[s][m]);  xn[m] = round(x[m] * r * w),
//   r = 1 / sqrt(mean(x[m]^2) + eps) over the rounded x ("Build your own
// Llama 3 from scratch" §3.6 residual, §3.1 RMSNorm).  One CTA of 1024 threads
// per row, 4*G consecutive-by-4 elements per thread held in registers; all
// of a thread's loads are issued before any of its stores.
template <int G>
__global__ void __launch_bounds__(1024) epi_residual_rmsnorm_kernel(const float* __restrict__ P, int splits,
                                                                   long long split_stride, bf16* __restrict__ x,
                                                                   const bf16* __restrict__ w,
                                                                   bf16* __restrict__ xn, int D, float eps) {
  griddep_wait_and_release();
  const int m = blockIdx.x;
  float v[G][4], r[G][4];
  float ss = 0.f;
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int n = 4 * (threadIdx.x + 1024 * g);
    if (n < D) {
      sum4_splits(P, splits, split_stride, (long long)m * D + n, v[g]);
      load4(x + (size_t)m * D + n, r[g]);
    }
  }
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int n = 4 * (threadIdx.x + 1024 * g);
    if (n < D) {
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        // round to bf16 exactly as the stored residual stream, then square that
        v[g][q] = __bfloat162float(__float2bfloat16_rn(v[g][q] + r[g][q]));
        ss = fmaf(v[g][q], v[g][q], ss);
      }
      store4(x + (size_t)m * D + n, v[g]);
    }
  }
  __shared__ float red[32];
  ss = warp_sum(ss);
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = ss;
  __syncthreads();
  float tot = 0.f;
#pragma unroll
  for (int i = 0; i < 32; ++i) tot += red[i];
  const float rs = rsqrtf(tot / (float)D + eps);
#pragma unroll
  for (int g = 0; g < G; ++g) {
    const int n = 4 * (threadIdx.x + 1024 * g);
    if (n < D) {
      float wv[4], o[4];
      load4(w + n, wv);
#pragma unroll
      for (int q = 0; q < 4; ++q) o[q] = v[g][q] * rs * wv[q];
      store4(xn + (size_t)m * D + n, o);
    }
  }
}

// g[m, f] = silu(P[m, f]) * P[m, F + f],  silu(z) = z / (1 + e^-z)
// ("Build your own Llama 3 from scratch" §3.5)
template <typename T>
__global__ void epi_swiglu_kernel(const float* __restrict__ P, int splits, long long split_stride,
                                  T* __restrict__ g, int M, int F) {
  griddep_wait_and_release();
  const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i >= (long long)M * F) return;
  const int m = (int)(i / F), f = (int)(i % F);
  float a[4], b[4], o[4];
  sum4_splits(P, splits, split_stride, (long long)m * 2 * F + f, a);
  sum4_splits(P, splits, split_stride, (long long)m * 2 * F + F + f, b);
#pragma unroll
  for (int q = 0; q < 4; ++q) o[q] = a[q] / (1.f + expf(-a[q])) * b[q];
  store4(g + i, o);
}

// QKV epilogue: rotate q and k pairs (2i, 2i+1) by the table's (cos, sin) of
// position start_pos + t ("Build your own Llama 3 from scratch" §3.2), write
// q to q_out [M, H*hd] and k, v to the caches at [b, pos, kvh, :] (§3.3).
// Two pairs (four elements, inside one head) per thread.
template <typename T>
__global__ void epi_qkv_rope_kernel(const float* __restrict__ P, int splits, long long split_stride,
                                    int M, int seq, int start_pos, int H, int KV, int hd,
                                    const float* __restrict__ rope, T* __restrict__ q_out,
                                    T* __restrict__ k_cache, T* __restrict__ v_cache, int cap,
                                    const int32_t* __restrict__ positions, int max_pos) {
  griddep_wait_and_release();
  const int Ntot = (H + 2 * KV) * hd;
  const long long i = ((long long)blockIdx.x * blockDim.x + threadIdx.x) * 4;
  if (i >= (long long)M * Ntot) return;
  const int m = (int)(i / Ntot);
  const int n = (int)(i % Ntot);
  const int b = m / seq, t = m % seq;
  int pos = start_pos + t;
  if (positions) {   // one token per sequence at its own position (out of range: flagged, clamped)
    pos = positions[b];
    if (pos < 0 || pos > max_pos) {
      if (n == 0) record_error(LLAMA3_ERR_ARG);
      pos = max(0, min(pos, max_pos));
    }
  }
  float v[4];
  sum4_splits(P, splits, split_stride, (long long)m * Ntot + n, v);
  const int d = n % hd, head = n / hd;
  if (head < H + KV) {
    const float4 cs = *reinterpret_cast<const float4*>(rope + ((size_t)pos * (hd / 2) + d / 2) * 2);
    const float a0 = v[0], b0 = v[1], a1 = v[2], b1 = v[3];
    v[0] = a0 * cs.x - b0 * cs.y;
    v[1] = a0 * cs.y + b0 * cs.x;
    v[2] = a1 * cs.z - b1 * cs.w;
    v[3] = a1 * cs.w + b1 * cs.z;
  }
  if (head < H) {
    store4(q_out + (size_t)m * H * hd + n, v);
  } else {
    const bool is_k = head < H + KV;
    const int kvh = head - (is_k ? H : H + KV);
    store4((is_k ? k_cache : v_cache) + (((size_t)b * cap + pos) * KV + kvh) * hd + d, v);
  }
}

// ---- causal GQA attention, one warp per (b, t, h) ---------------------------
// ("Build your own Llama 3 from scratch" §3.4; query head h reads KV head
// h / (H/KV); key j is visible to position start_pos + t iff j <= start_pos + t)
// Online softmax in fp32.  Lane l owns dims l, l+32, ... of the output.
template <typename T>
__global__ void attention_simt_kernel(const T* __restrict__ q, const T* __restrict__ k_cache,
                                      const T* __restrict__ v_cache, T* __restrict__ out, int B,
                                      int S, int start_pos, int H, int KV, int hd, int cap,
                                      float scale, const int32_t* __restrict__ doc_start,
                                      const int32_t* __restrict__ positions, int max_pos) {
  griddep_wait_and_release();
  long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (w >= (long long)B * S * H) return;
  int h = (int)(w % H);
  int t = (int)((w / H) % S);
  int b = (int)(w / ((long long)H * S));
  int g = h / (H / KV);
  const T* qr = q + (((size_t)b * S + t) * H + h) * hd;
  float qv[4], acc[4];
  for (int i = 0; i < 4; ++i) {
    int d = lane + 32 * i;
    qv[i] = d < hd ? to_f(qr[d]) : 0.f;
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  // per-sequence positions (one token per sequence): clamped into range
  const int last = positions ? max(0, min(positions[b], max_pos)) : start_pos + t;
  // document mask: keys before the start of this token's document are invisible
  const int first = doc_start ? max(0, min(doc_start[(size_t)b * S + t], last)) : 0;
  for (int j = first; j <= last; ++j) {
    const T* kr = k_cache + (((size_t)b * cap + j) * KV + g) * hd;
    const T* vr = v_cache + (((size_t)b * cap + j) * KV + g) * hd;
    float s = 0.f;
    for (int i = 0; i < 4; ++i) {
      int d = lane + 32 * i;
      if (d < hd) s = fmaf(qv[i], to_f(kr[d]), s);
    }
    s = warp_sum(s) * scale;
    float mn = fmaxf(m, s);
    float corr = expf(m - mn);  // exp(-inf) = 0 on the first key
    float p = expf(s - mn);
    l = l * corr + p;
    for (int i = 0; i < 4; ++i) {
      int d = lane + 32 * i;
      acc[i] = acc[i] * corr + (d < hd ? p * to_f(vr[d]) : 0.f);
    }
    m = mn;
  }
  T* orow = out + (((size_t)b * S + t) * H + h) * hd;
  float inv = 1.f / l;
  for (int i = 0; i < 4; ++i) {
    int d = lane + 32 * i;
    if (d < hd) orow[d] = from_f<T>(acc[i] * inv);
  }
}

// ---- LM head: logits and argmax ("llama3-from-scratch：输出层与预测") --------
// One warp per (row r, block of 32 vocabulary rows); one atomicMax per warp.
template <typename T>
__global__ void lm_head_simt_kernel(const T* __restrict__ hn, const T* __restrict__ W,
                                    float* __restrict__ logits, unsigned long long* __restrict__ keys,
                                    int R, int V, int D) {
  griddep_wait_and_release();
  long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  int vblocks = (V + 31) / 32;
  if (w >= (long long)R * vblocks) return;
  int r = (int)(w / vblocks);
  int v0 = (int)(w % vblocks) * 32;
  const T* hr = hn + (size_t)r * D;
  unsigned long long best = 0;
  for (int v = v0; v < min(v0 + 32, V); ++v) {
    const T* wr = W + (size_t)v * D;
    float s = 0.f;
    for (int i = lane; i < D; i += 32) s = fmaf(to_f(hr[i]), to_f(wr[i]), s);
    s = warp_sum(s);
    if (logits && lane == 0) logits[(size_t)r * V + v] = s;
    unsigned long long k = argmax_pack(s, (uint32_t)v);
    best = k > best ? k : best;
  }
  if (lane == 0) atomicMax(&keys[r], best);
}

__global__ void argmax_init_kernel(unsigned long long* keys, int R) {
  griddep_wait_and_release();
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < R) keys[i] = 0ull;
}
__global__ void argmax_finalize_kernel(const unsigned long long* keys, int32_t* ids, int R) {
  griddep_wait_and_release();
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < R) ids[i] = (int32_t)(0xffffffffu - (uint32_t)(keys[i] & 0xffffffffull));
}

}  // namespace l3
