// sampling.cuh -- temperature / top-p draw of the next token on the device.
//
// What it computes ("Build your own Llama 3 from scratch" 六, generate and
// sample_top_p): for one row of fp32 logits l and temperature T > 0,
//   p = softmax(l / T); rank tokens by descending p (ties: lower index first);
//   keep a token iff the probability ranked before it is <= top_p;
//   renormalise over the kept tokens and draw one.
// T <= 0 takes the argmax (lowest index on ties), as the page does for T = 0.
//
// Device formulation (one CTA of 1024 threads per row; no sort):
//  * e_v = exp(l_v / T - max) in fp32, carried as an integer mass
//    f_v = round(e_v * 2^40) (the largest e is 1, so the row total is below
//    2^58).  Integer sums are exact and order-free, so every decision below is
//    deterministic.  The rank order is the order of the fp32 bit pattern of
//    e_v (positive floats sort like unsigned integers), then the index.
//  * The kept set is a prefix of the rank order ending at the first token b
//    whose inclusive ranked mass exceeds thr = floor(top_p * total).  b's key
//    is found by a most-significant-digit radix select (four 8-bit digits)
//    over per-warp mass histograms in shared memory; the tokens tied with b
//    are kept up to the needed count in index order.
//  * The draw: word = first output of Philox-4x64-10 (Salmon et al., "Parallel
//    random numbers: as easy as 1, 2, 3", SC 2011) with key (seed, 0) and
//    counter (offset [+ positions[row]], row, 0, 0); target = floor(word * K / 2^64) for the kept
//    mass K; the token is the first kept one, in index order, whose running
//    kept mass exceeds target (the inverse CDF of the renormalised kept law).
#pragma once
#include "common.cuh"

namespace l3 {

struct SampleParams {
  const float* logits;
  long long ld;
  int V;
  float temperature, top_p;
  unsigned long long seed, offset;
  const int32_t* positions;   // optional: row r's draw counts from offset + positions[r]
  int32_t* ids;
};

// Philox-4x64-10 block; only the first output word is used.
__device__ __forceinline__ uint64_t philox4x64_10_word0(uint64_t c0, uint64_t c1, uint64_t c2, uint64_t c3,
                                                        uint64_t k0, uint64_t k1) {
  const uint64_t mul0 = 0xD2E7470EE14C6C93ull, mul1 = 0xCA5A826395121157ull;
  const uint64_t weyl0 = 0x9E3779B97F4A7C15ull, weyl1 = 0xBB67AE8584CAA73Bull;
#pragma unroll 1
  for (int r = 0; r < 10; ++r) {
    const uint64_t hi0 = __umul64hi(mul0, c0), lo0 = mul0 * c0;
    const uint64_t hi1 = __umul64hi(mul1, c2), lo1 = mul1 * c2;
    const uint64_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0; c1 = lo1; c2 = n2; c3 = lo0;
    k0 += weyl0; k1 += weyl1;
  }
  return c0;
}

constexpr int kSampleThreads = 1024;
constexpr int kSampleWarps = kSampleThreads / 32;
constexpr int kSampleSmem = kSampleWarps * 256 * 8;   // per-warp 256-bucket mass histograms

__device__ __forceinline__ float sample_scaled(const float* lg, int v, float T) { return __fdiv_rn(lg[v], T); }
__device__ __forceinline__ float sample_e(const float* lg, int v, float T, float zmax) {
  return expf(sample_scaled(lg, v, T) - zmax);
}
__device__ __forceinline__ uint64_t sample_mass(float e) { return __float2ull_rn(e * 1099511627776.0f); }

__device__ __forceinline__ uint64_t warp_sum_u64(uint64_t v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ uint64_t warp_incl_scan_u64(uint64_t v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

__global__ void __launch_bounds__(kSampleThreads) sample_top_p_kernel(const SampleParams sp) {
  griddep_wait_and_release();
  extern __shared__ uint64_t hist[];   // [warp][256]
  __shared__ float s_f[kSampleWarps];
  __shared__ int s_i[kSampleWarps];
  __shared__ uint64_t s_u[kSampleWarps], s_u2[kSampleWarps];
  __shared__ uint64_t s_bucket[256];
  __shared__ uint32_t s_prefix;
  __shared__ uint64_t s_above;
  __shared__ int s_pick;

  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* lg = sp.logits + (size_t)row * sp.ld;
  const int V = sp.V;
  const float T = sp.temperature;

  // ---- greedy: argmax, lowest index on ties
  if (!(T > 0.f)) {
    float best = -INFINITY;
    int bi = 0x7fffffff;
    for (int v = tid; v < V; v += kSampleThreads) {
      const float x = lg[v];
      if (x > best || (x == best && v < bi)) { best = x; bi = v; }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ob = __shfl_xor_sync(0xffffffffu, best, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ob > best || (ob == best && oi < bi)) { best = ob; bi = oi; }
    }
    if (lane == 0) { s_f[warp] = best; s_i[warp] = bi; }
    __syncthreads();
    if (tid == 0) {
      float b = s_f[0];
      int i = s_i[0];
      for (int w = 1; w < kSampleWarps; ++w)
        if (s_f[w] > b || (s_f[w] == b && s_i[w] < i)) { b = s_f[w]; i = s_i[w]; }
      sp.ids[row] = (i < V) ? i : 0;
    }
    return;
  }

  // ---- max of the scaled logits
  float zmax = -INFINITY;
  for (int v = tid; v < V; v += kSampleThreads) zmax = fmaxf(zmax, sample_scaled(lg, v, T));
  zmax = warp_max(zmax);
  if (lane == 0) s_f[warp] = zmax;
  __syncthreads();
  zmax = s_f[0];
#pragma unroll 1
  for (int w = 1; w < kSampleWarps; ++w) zmax = fmaxf(zmax, s_f[w]);

  // ---- total mass
  uint64_t tot = 0;
  for (int v = tid; v < V; v += kSampleThreads) tot += sample_mass(sample_e(lg, v, T, zmax));
  tot = warp_sum_u64(tot);
  if (lane == 0) s_u[warp] = tot;
  __syncthreads();
  uint64_t total = 0;
#pragma unroll 1
  for (int w = 0; w < kSampleWarps; ++w) total += s_u[w];
  __syncthreads();   // every thread has read s_u before pass A reuses it

  const double pt = (double)sp.top_p * (double)total;
  const bool keep_all = !(pt < (double)total);
  const uint64_t thr = keep_all ? total : (uint64_t)pt;

  // ---- radix select of b's key: A = mass ranked strictly above the current bucket
  uint32_t prefix = 0;
  uint64_t above = 0;
  if (!keep_all) {
#pragma unroll 1
    for (int level = 0; level < 4; ++level) {
      const int shift = 24 - 8 * level;
      const uint32_t hi_mask = level == 0 ? 0u : (0xffffffffu << (shift + 8));
      uint64_t* h = hist + warp * 256;
      for (int d = lane; d < 256; d += 32) h[d] = 0;
      __syncwarp();
      for (int v = tid; v < V; v += kSampleThreads) {
        const float e = sample_e(lg, v, T, zmax);
        const uint32_t key = __float_as_uint(e);
        if ((key & hi_mask) == prefix) atomicAdd(reinterpret_cast<unsigned long long*>(&h[(key >> shift) & 255u]),
                                                 (unsigned long long)sample_mass(e));
      }
      __syncthreads();
      if (tid < 256) {
        uint64_t m = 0;
#pragma unroll 4
        for (int w = 0; w < kSampleWarps; ++w) m += hist[w * 256 + tid];
        s_bucket[tid] = m;
      }
      __syncthreads();
      if (warp == 0) {
        // lane l owns digits 255-8l down to 248-8l (descending rank order)
        uint64_t mine = 0;
#pragma unroll
        for (int q = 0; q < 8; ++q) mine += s_bucket[255 - 8 * lane - q];
        const uint64_t incl = warp_incl_scan_u64(mine, lane);
        const uint64_t excl = incl - mine;
        const unsigned cross = __ballot_sync(0xffffffffu, above + incl > thr);
        const int first = cross ? __ffs(cross) - 1 : 31;
        if (lane == first) {
          uint64_t acc = above + excl;
          int d = 255 - 8 * lane;
          for (int q = 0; q < 8; ++q, --d) {
            const uint64_t m = s_bucket[d];
            if (acc + m > thr || q == 7) break;
            acc += m;
          }
          s_prefix = prefix | ((uint32_t)d << shift);
          s_above = acc;
        }
      }
      __syncthreads();
      prefix = s_prefix;
      above = s_above;
    }
  }

  // ---- kept set: keys > kb, plus the first n_tie tokens (index order) with key == kb
  const uint32_t kb = prefix;
  uint64_t fb = 0, n_tie = 0, kept_mass = total;
  if (!keep_all) {
    fb = sample_mass(__uint_as_float(kb));
    n_tie = fb ? (thr - above) / fb + 1 : 0;
    kept_mass = above + n_tie * fb;
  }
  const uint64_t ctr = sp.offset + (sp.positions ? (uint64_t)(int64_t)sp.positions[row] : 0ull);
  const uint64_t word = philox4x64_10_word0(ctr, (uint64_t)row, 0, 0, sp.seed, 0);
  const uint64_t target = __umul64hi(word, kept_mass);

  // ---- pass A: per-warp segment totals (warp w owns indices [w*seg, (w+1)*seg))
  const int seg = ((V + kSampleWarps - 1) / kSampleWarps + 31) & ~31;
  const int s0 = min(V, warp * seg), s1 = min(V, s0 + seg);
  uint64_t g_mass = 0, ties = 0;
  for (int v = s0 + lane; v < s1; v += 32) {
    const float e = sample_e(lg, v, T, zmax);
    const uint32_t key = __float_as_uint(e);
    if (keep_all || key > kb) g_mass += sample_mass(e);
    else if (key == kb) ties += 1;
  }
  g_mass = warp_sum_u64(g_mass);
  ties = warp_sum_u64(ties);
  if (lane == 0) { s_u[warp] = g_mass; s_u2[warp] = ties; }
  if (tid == 0) s_pick = -1;
  __syncthreads();
  // the warp whose segment holds the target walks it
  uint64_t tie0 = 0, mass0 = 0;
#pragma unroll 1
  for (int w = 0; w < warp; ++w) {
    const uint64_t kt = s_u2[w] < (n_tie > tie0 ? n_tie - tie0 : 0) ? s_u2[w] : (n_tie > tie0 ? n_tie - tie0 : 0);
    mass0 += s_u[w] + kt * fb;
    tie0 += s_u2[w];
  }
  const uint64_t my_kt_cap = n_tie > tie0 ? n_tie - tie0 : 0;
  const uint64_t my_kept = g_mass + (ties < my_kt_cap ? ties : my_kt_cap) * fb;
  const bool mine = (mass0 <= target && target < mass0 + my_kept) || (warp == kSampleWarps - 1 && target >= mass0 + my_kept);
  if (mine && s0 < s1) {
    uint64_t run = mass0, tie_run = tie0;
    int pick = -1;
    for (int base = s0; base < s1 && pick < 0; base += 32) {
      const int v = base + lane;
      uint64_t f = 0;
      bool tie = false;
      if (v < s1) {
        const float e = sample_e(lg, v, T, zmax);
        const uint32_t key = __float_as_uint(e);
        if (keep_all || key > kb) f = sample_mass(e);
        else if (key == kb) tie = true;
      }
      const unsigned tmask = __ballot_sync(0xffffffffu, tie);
      const uint64_t rank = tie_run + __popc(tmask & ((1u << lane) - 1u));
      if (tie && rank < n_tie) f = fb;
      const uint64_t incl = warp_incl_scan_u64(f, lane) + run;
      const unsigned hit = __ballot_sync(0xffffffffu, f > 0 && incl > target);
      if (hit) pick = base + __ffs(hit) - 1;
      run = __shfl_sync(0xffffffffu, incl, 31);
      tie_run += __popc(tmask);
    }
    if (lane == 0 && pick >= 0) s_pick = pick;
  }
  __syncthreads();
  if (tid == 0) {
    int pick = s_pick;
    if (pick < 0) pick = 0;   // unreachable for a finite row: target < kept mass
    sp.ids[row] = pick;
  }
}

}  // namespace l3
