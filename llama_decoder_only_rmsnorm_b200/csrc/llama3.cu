// llama3.cu -- host side of the C ABI declared in include/llama3.h.
//
// One translation unit: it includes every kernel header so that the device
// status word and the kernels live in one module.  Entry points validate
// every argument before launching anything, build TMA descriptors for the
// tcgen05 kernels, carve the caller's workspace, and launch on the caller's
// stream.  No device memory is allocated here.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "decode_attention.cuh"
#include "flash_attention.cuh"
#include "sampling.cuh"
#include "simt.cuh"
#include "tc_gemm.cuh"
#include "tc_gemm_pair.cuh"

using namespace l3;

namespace {

thread_local int t_last_cuda = 0;
int g_kernel_path = 0;       // 0 = tcgen05 for bf16, 1 = SIMT everywhere
// Prefill GEMMs run on CTA pairs (tc_gemm_pair.cuh) once there are at least
// 256 token rows: on the 8B prefill step that measured 107.1 against 109.2 ms
// with single-CTA tiles (interleaved runs on one box), bit-identical results.
bool use_pair_gemm(int m) { return m >= 256; }
int g_wait_ms = 2000;        // bounded device waits
int g_withhold = 0;          // failure-detection test hook (llama3_set_test_withheld_arrival)
constexpr int kMaxDevices = 64;
int g_num_sms[kMaxDevices];

int cuda_fail(cudaError_t e) {
  t_last_cuda = (int)e;
  return LLAMA3_ERR_CUDA;
}
#define L3_CUDA(call)                            \
  do {                                           \
    cudaError_t e_ = (call);                     \
    if (e_ != cudaSuccess) return cuda_fail(e_); \
  } while (0)
#define L3_TRY(call)              \
  do {                            \
    int s_ = (call);              \
    if (s_ != LLAMA3_OK) return s_; \
  } while (0)

int launch_check() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? LLAMA3_OK : cuda_fail(e);
}

// Launch accounting and the optional per-family event timer.
std::atomic<unsigned long long> g_launches{0};
struct LaunchTimer {
  int kind = 0, n = 0, used = 0;
  std::vector<cudaEvent_t> start, stop;
} g_timer;

// Inside a stream capture the record must become an external event node so
// that every replay of the graph timestamps the event.
void timer_record(cudaEvent_t ev, cudaStream_t st) {
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cs) == cudaSuccess && cs == cudaStreamCaptureStatusActive)
    cudaEventRecordWithFlags(ev, st, cudaEventRecordExternal);
  else
    cudaEventRecord(ev, st);
}
void timer_begin(int kind, cudaStream_t st) {
  if (g_timer.kind == kind && g_timer.used < g_timer.n) timer_record(g_timer.start[g_timer.used], st);
}
void timer_end(int kind, cudaStream_t st) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  if (g_timer.kind == kind && g_timer.used < g_timer.n) timer_record(g_timer.stop[g_timer.used++], st);
}
// Launch `call` (a launch_k(...) expression) as family `kind` on `st`.
#define L3_LAUNCH(kind, st, ...)                        \
  do {                                                  \
    timer_begin((kind), (st));                          \
    const cudaError_t le_ = (__VA_ARGS__);              \
    timer_end((kind), (st));                            \
    if (le_ != cudaSuccess) return cuda_fail(le_);      \
  } while (0)

// Kernels are launched with programmatic stream serialization: one may be
// scheduled while its predecessor in the stream finishes, and it waits for
// that predecessor (griddepcontrol.wait) after its own set-up and before it
// touches memory.  g_pdl = false launches them all the ordinary way.  The
// prefill GEMMs that follow an RMSNorm launch the ordinary way in any case:
// on B200, letting their CTAs in while the norm runs made the 8B prefill step
// 3-4 % slower (112.7-115.8 against 109.1-111.6 ms in interleaved runs on two
// boxes), while every other kernel gains or is neutral.
bool g_pdl = true;

template <typename... KArgs, typename... Args>
cudaError_t launch_k_pdl(bool pdl, void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                         Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = (g_pdl && pdl) ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}
template <typename... KArgs, typename... Args>
cudaError_t launch_k(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                     Args... args) {
  return launch_k_pdl(true, kern, grid, block, smem, st, args...);
}

int current_device(int* dev) {
  cudaError_t e = cudaGetDevice(dev);
  if (e != cudaSuccess) return cuda_fail(e);
  if (*dev < 0 || *dev >= kMaxDevices) return LLAMA3_ERR_UNSUPPORTED;
  return LLAMA3_OK;
}

int num_sms() {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return 148;
  if (!g_num_sms[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    g_num_sms[dev] = n;
  }
  return g_num_sms[dev];
}

unsigned long long wait_ns() { return (unsigned long long)g_wait_ms * 1000000ull; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

size_t esize(const llama3_config* c) { return c->dtype == LLAMA3_DTYPE_F32 ? 4 : 2; }

// tcgen05/TMA kernels: bf16 with head_dim >= 64 (their RoPE epilogue rotates
// 32-column chunks inside one head); smaller heads run on the SIMT kernels.
bool use_tc(const llama3_config* c) {
  return c->dtype == LLAMA3_DTYPE_BF16 && g_kernel_path != 1 && c->head_dim >= 64;
}

int check_config(const llama3_config* c) {
  if (!c) return LLAMA3_ERR_ARG;
  if (c->dtype != LLAMA3_DTYPE_BF16 && c->dtype != LLAMA3_DTYPE_F32) return LLAMA3_ERR_ARG;
  if (c->dim < 1 || c->n_heads < 1 || c->n_kv_heads < 1 || c->head_dim < 2) return LLAMA3_ERR_ARG;
  if (c->n_heads % c->n_kv_heads) return LLAMA3_ERR_ARG;
  if (c->dim != c->n_heads * c->head_dim) return LLAMA3_ERR_ARG;
  const int hd = c->head_dim;
  if (hd != 16 && hd != 32 && hd != 64 && hd != 96 && hd != 128) return LLAMA3_ERR_ARG;
  if (c->ffn_hidden < 1 || c->vocab < 0) return LLAMA3_ERR_ARG;
  if (!(c->norm_eps > 0.f) || !(c->rope_theta > 1.0)) return LLAMA3_ERR_ARG;
  if (c->dtype == LLAMA3_DTYPE_BF16) {
    if (c->dim % 8 || c->ffn_hidden % 8) return LLAMA3_ERR_ARG;
  } else if (c->dim % 4 || c->ffn_hidden % 4) {
    return LLAMA3_ERR_ARG;
  }
  return LLAMA3_OK;
}

// ---------------------------------------------------------------------------
// TMA descriptors (driver entry point fetched through the runtime, so the
// library does not link libcuda directly)
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;
std::once_flag g_encode_once;

int encode_fn(EncodeTiledFn* fn) {
  std::call_once(g_encode_once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<EncodeTiledFn>(p);
  });
  *fn = g_encode;
  return g_encode ? LLAMA3_OK : LLAMA3_ERR_CUDA;
}

// bf16 matrix [rows, cols] row-major, box of 64 columns x box_rows rows,
// 128-byte swizzle; out-of-range elements read as zero.
int make_map(CUtensorMap* m, const void* ptr, long long rows, long long cols, int box_rows) {
  EncodeTiledFn enc;
  L3_TRY(encode_fn(&enc));
  if (!aligned16(ptr) || (cols * 2) % 16) return LLAMA3_ERR_ALIGN;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
  cuuint32_t es[2] = {1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_cuda = (int)r;
    return LLAMA3_ERR_CUDA;
  }
  return LLAMA3_OK;
}

// bf16 4-D tensor {d0 (contiguous), d1, d2, d3} with byte strides for d1..d3,
// box {64, 1, 128, 1}, 128-byte swizzle (one 128-row slab of 64 elements).
int make_map_4d(CUtensorMap* m, const void* ptr, long long d0, long long d1, long long d2, long long d3,
                long long s1_bytes, long long s2_bytes, long long s3_bytes) {
  EncodeTiledFn enc;
  L3_TRY(encode_fn(&enc));
  if (!aligned16(ptr) || s1_bytes % 16 || s2_bytes % 16 || s3_bytes % 16) return LLAMA3_ERR_ALIGN;
  cuuint64_t dims[4] = {(cuuint64_t)d0, (cuuint64_t)d1, (cuuint64_t)d2, (cuuint64_t)d3};
  cuuint64_t strides[3] = {(cuuint64_t)s1_bytes, (cuuint64_t)s2_bytes, (cuuint64_t)s3_bytes};
  cuuint32_t box[4] = {64u, 1u, 128u, 1u};
  cuuint32_t es[4] = {1u, 1u, 1u, 1u};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    t_last_cuda = (int)r;
    return LLAMA3_ERR_CUDA;
  }
  return LLAMA3_OK;
}

bool flash_attention_supported(int hd, int H, int KV) {
  (void)H; (void)KV;
  return hd == 64 || hd == 96 || hd == 128;
}

template <int HD>
int run_flash_attention_t(int H, int KV, const void* q, const void* kc, const void* vc, int cap, int B, int S,
                          int P, void* out, const int32_t* doc_start, int sms, unsigned long long wns,
                          cudaStream_t st) {
  CUtensorMap mq, mk, mv;
  const long long e = 2;
  L3_TRY(make_map_4d(&mq, q, HD, H, S, B, HD * e, (long long)H * HD * e, (long long)S * H * HD * e));
  L3_TRY(make_map_4d(&mk, kc, HD, KV, P + S, B, HD * e, (long long)KV * HD * e, (long long)cap * KV * HD * e));
  L3_TRY(make_map_4d(&mv, vc, HD, KV, P + S, B, HD * e, (long long)KV * HD * e, (long long)cap * KV * HD * e));
  FlashShape fs;
  fs.B = B; fs.S = S; fs.P = P; fs.H = H; fs.KV = KV;
  fs.n_rep = H / KV;
  fs.pairs = (fs.n_rep + 1) / 2;
  fs.qtiles = (S + 127) / 128;
  fs.units = B * KV * fs.pairs * fs.qtiles;
  fs.ldo = H * HD;
  fs.scale_log2 = (float)(1.4426950408889634 / sqrt((double)HD));
  fs.doc_start = doc_start;
  fs.withhold = g_withhold == 2 ? 2 : 0;
  constexpr int smem = FlashCfg<HD>::SMEM_BYTES;
  auto kern = flash_attention_kernel<HD>;
  int dev = 0;
  L3_TRY(current_device(&dev));
  static bool attr_done[kMaxDevices];
  static bool regs_ok[kMaxDevices];
  if (!attr_done[dev]) {
    L3_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
    // The warpgroups' setmaxnreg shares must fit the registers the block is
    // launched with, or the raising warpgroups would wait for ever.
    cudaFuncAttributes fa;
    L3_CUDA(cudaFuncGetAttributes(&fa, kern));
    regs_ok[dev] = (long long)fa.numRegs * kFlashThreads >= 128LL * kFlashLowRegs + 256LL * kFlashHighRegs;
    attr_done[dev] = true;
  }
  if (!regs_ok[dev]) return LLAMA3_ERR_UNSUPPORTED;
  const int grid = std::min(fs.units, sms);
  L3_LAUNCH(LLAMA3_KERNEL_ATTENTION, st,
            launch_k(kern, grid, kFlashThreads, smem, st, mq, mk, mv, (bf16*)out, fs, wns));
  return launch_check();
}

int run_flash_attention(int hd, int H, int KV, const void* q, const void* kc, const void* vc, int cap, int B, int S,
                        int P, void* out, const int32_t* doc_start, int sms, unsigned long long wns,
                        cudaStream_t st) {
  switch (hd) {
    case 64: return run_flash_attention_t<64>(H, KV, q, kc, vc, cap, B, S, P, out, doc_start, sms, wns, st);
    case 96: return run_flash_attention_t<96>(H, KV, q, kc, vc, cap, B, S, P, out, doc_start, sms, wns, st);
    case 128: return run_flash_attention_t<128>(H, KV, q, kc, vc, cap, B, S, P, out, doc_start, sms, wns, st);
    default: return LLAMA3_ERR_UNSUPPORTED;
  }
}

// ---------------------------------------------------------------------------
// Workspace layout
// ---------------------------------------------------------------------------
constexpr int kMaxSplitK = 16;
constexpr int kMaxKvSplits = 128;

struct Workspace {
  size_t xn, q, o, g, part, attn_part, lm_rows, keys, total;
};

size_t up256(size_t x) { return (x + 255) & ~size_t(255); }

Workspace layout(const llama3_config* c, int batch, int seq, int lm_rows) {
  Workspace w;
  const size_t es = esize(c);
  const size_t M = (size_t)batch * seq;
  const int H = c->n_heads, KV = c->n_kv_heads, hd = c->head_dim, D = c->dim, F = c->ffn_hidden;
  const size_t nqkv = (size_t)(H + 2 * KV) * hd;
  const size_t widest = std::max(nqkv, std::max((size_t)D, (size_t)2 * F));
  size_t off = 0;
  w.xn = off; off += up256(M * D * es);
  w.q = off; off += up256(M * H * hd * es);
  w.o = off; off += up256(M * H * hd * es);
  w.g = off; off += up256(M * F * es);
  // fp32 partial sums: whole [M, widest] for the SIMT path; kMaxSplitK slabs of
  // [batch, widest] for the split-K decode GEMMs.
  size_t part = kMaxSplitK * (size_t)batch * widest * 4;
  if (!use_tc(c)) part = std::max(part, M * widest * 4);
  w.part = off; off += up256(part);
  w.attn_part = off; off += up256((size_t)batch * H * kMaxKvSplits * (hd + 2) * 4);
  const size_t R = (size_t)std::max(lm_rows, 1);
  w.lm_rows = off; off += up256(R * D * es);
  w.keys = off; off += up256(R * 8);
  w.total = off;
  return w;
}

template <typename T>
T* ws_at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

// ---------------------------------------------------------------------------
// tcgen05 GEMM launch helpers
// ---------------------------------------------------------------------------
#ifndef L3_GROUP_M
#define L3_GROUP_M 32
#endif
GemmShape make_shape(int rows_a, int rows_a2, int rows_b, int k, int bn, int splits) {
  GemmShape s;
  s.rows_a = rows_a;
  s.rows_a2 = rows_a2;
  s.rows_b = rows_b;
  s.k = k;
  s.tiles_m1 = (rows_a + 127) / 128;
  s.tiles_m = s.tiles_m1 + (rows_a2 + 127) / 128;
  s.tiles_n = (rows_b + bn - 1) / bn;
  s.kblocks = (k + 63) / 64;
  splits = std::max(1, std::min(splits, s.kblocks));
  s.kb_per_split = (s.kblocks + splits - 1) / splits;
  s.splits = (s.kblocks + s.kb_per_split - 1) / s.kb_per_split;
  s.units = s.splits * s.tiles_m * s.tiles_n;
  // Groups of L3_GROUP_M m-tiles: with a 148-CTA persistent grid the tiles in
  // flight span that many A row-blocks x ~148/L3_GROUP_M B column-blocks
  // (32 measured best on the 8B prefill: the step ran at a higher clock than
  // with 16, and 64 lowered the clock).  The
  // swapped (weight-streaming) launches have one n-tile, where grouping
  // changes nothing.
  s.group_m = std::max(1, std::min(L3_GROUP_M, s.tiles_m));
  s.sk_per = 0;
  s.withhold = 0;
  return s;
}

// Split count that minimises the longest per-CTA stream (persistent grid of
// one CTA per SM): ceil(units / SMs) * k-blocks per split.
// Split-K count for a skinny GEMM: minimise the busiest CTA's load, counted
// in k-blocks, where every work unit also costs L3_SPLIT_UNIT_COST k-blocks
// for writing its fp32 partial tile and reading it back in the reduction.
#ifndef L3_SPLIT_UNIT_COST
#define L3_SPLIT_UNIT_COST 2
#endif
// Stream-K plan for `tiles` tiles of `kblocks` k-blocks on `sms` CTAs: per =
// k-blocks per CTA, ctas = CTAs with work, slabs = most CTAs sharing a tile,
// cost = the busiest CTA's k-blocks plus L3_SPLIT_UNIT_COST per tile it
// touches (the same units as choose_splits).
struct StreamK {
  bool ok;
  int per, ctas, slabs;
  long long cost;
};
StreamK plan_stream_k(int tiles, int kblocks, int sms) {
  StreamK p{};
  const long long total = (long long)tiles * kblocks;
  if (total <= 0 || sms <= 0) return p;
  p.per = (int)((total + sms - 1) / sms);
  p.ctas = (int)((total + p.per - 1) / p.per);
  int slabs = 0, most_units = 0;
  for (int t = 0; t < tiles; ++t) {
    const long long t0 = (long long)t * kblocks;
    slabs = std::max(slabs, (int)((t0 + kblocks - 1) / p.per - t0 / p.per + 1));
  }
  for (int c = 0; c < p.ctas; ++c) {
    const long long a = (long long)c * p.per, b = std::min(a + p.per, total);
    most_units = std::max(most_units, (int)((b - 1) / kblocks - a / kblocks + 1));
  }
  p.slabs = slabs;
  p.cost = p.per + (long long)most_units * L3_SPLIT_UNIT_COST;
  p.ok = slabs <= kMaxSplitK;
  return p;
}

int choose_splits(int tiles, int kblocks, int sms) {
  int best = 1;
  long long best_t = -1;
  for (int s = 1; s <= std::min(kMaxSplitK, kblocks); ++s) {
    const int per = (kblocks + s - 1) / s;
    const int real = (kblocks + per - 1) / per;
    const long long units = (long long)tiles * real;
    const long long t = ((units + sms - 1) / sms) * (per + L3_SPLIT_UNIT_COST);
    if (best_t < 0 || t < best_t) { best_t = t; best = real; }
  }
  return best;
}

template <int BN, int STAGES, int EPI, bool DUAL>
int launch_gemm(int kind, const CUtensorMap& a, const CUtensorMap& a2, const CUtensorMap& b, const CUtensorMap& b2,
                const GemmShape& sh, const EpiParams& ep, cudaStream_t st) {
  using Cfg = TcGemmCfg<BN, STAGES, DUAL>;
  auto kern = tc_gemm_kernel<BN, STAGES, EPI, DUAL>;
  int dev = 0;
  L3_TRY(current_device(&dev));
  static bool attr_done[kMaxDevices];
  if (!attr_done[dev]) {
    L3_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES));
    attr_done[dev] = true;
  }
  if (sh.units <= 0) return LLAMA3_OK;
  const int grid = std::min(sh.units, num_sms());
  GemmShape s = sh;
  s.withhold = g_withhold == 1 ? 1 : 0;
  const bool after_norm = kind == LLAMA3_KERNEL_GEMM_QKV || kind == LLAMA3_KERNEL_GEMM_W13;
  L3_LAUNCH(kind, st, launch_k_pdl(!after_norm, kern, grid, 192, Cfg::SMEM_BYTES, st, a, a2, b, b2, s, ep, wait_ns()));
  return launch_check();
}

// Prefill GEMM shape for CTA pairs: 256-row tiles of A, raster groups of 16
// of them (the same 4096 rows as the single-CTA raster's 32 tiles of 128).
GemmShape make_shape_pair(int rows_a, int rows_b, int k, int bn) {
  GemmShape s = make_shape(rows_a, 0, rows_b, k, bn, 1);
  s.tiles_m1 = s.tiles_m = (rows_a + 255) / 256;
  s.units = s.tiles_m * s.tiles_n;
  s.group_m = std::max(1, std::min(L3_GROUP_M / 2, s.tiles_m));
  return s;
}

template <int BN, int STAGES, int EPI, bool DUAL>
int launch_gemm_pair(int kind, const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b2,
                     const GemmShape& sh, const EpiParams& ep, cudaStream_t st) {
  using Cfg = TcGemmPairCfg<BN, STAGES, DUAL>;
  auto kern = tc_gemm_pair_kernel<BN, STAGES, EPI, DUAL>;
  int dev = 0;
  L3_TRY(current_device(&dev));
  static bool attr_done[kMaxDevices];
  if (!attr_done[dev]) {
    L3_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES));
    attr_done[dev] = true;
  }
  if (sh.units <= 0) return LLAMA3_OK;
  GemmShape s = sh;
  s.withhold = g_withhold == 1 ? 1 : 0;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(192);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // One persistent pair per cluster slot the device can hold at once (two SMs
  // of one GPC each); pairs never wait on one another, so a smaller count
  // would only be slower, never stuck.
  static int max_pairs[kMaxDevices];
  if (!max_pairs[dev]) {
    cfg.gridDim = dim3(2 * std::max(1, num_sms() / 2));
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, kern, &cfg) != cudaSuccess || n < 1) {
      (void)cudaGetLastError();   // a failed query must not be reported as the launch's error
      n = std::max(1, num_sms() / 2);
    }
    max_pairs[dev] = std::min(n, std::max(1, num_sms() / 2));
  }
  const int pairs = std::min(s.units, max_pairs[dev]);
  cfg.gridDim = dim3(2 * pairs);
  const bool after_norm = kind == LLAMA3_KERNEL_GEMM_QKV || kind == LLAMA3_KERNEL_GEMM_W13;
  cfg.numAttrs = (g_pdl && !after_norm) ? 2 : 1;
  const unsigned long long wns = wait_ns();
  L3_LAUNCH(kind, st, cudaLaunchKernelEx(&cfg, kern, a, b, b2, s, ep, wns));
  return launch_check();
}

EpiParams empty_epi() {
  EpiParams e;
  memset(&e, 0, sizeof(e));
  return e;
}

// Swapped (weight-streaming) GEMM for few token rows: P[split][t][n] =
// sum_k W[n, k] X[t, k], with W1|W3 stacked through `w_second`.
// Skinny GEMM with the weights as the MMA's M side and split-K: fp32 partials
// P[split][token][feature], reduced by a separate kernel.
// Schedule of a weight-streaming GEMM: rows_w (+ rows_w2 stacked) weight rows
// as the MMA M side, rows_x tokens as N (tile width bn), k deep.
GemmShape plan_swapped(int rows_w, int rows_w2, int rows_x, int k, int bn) {
  const int tiles = ((rows_w + 127) / 128 + (rows_w2 + 127) / 128) * ((rows_x + bn - 1) / bn);
  const int kblocks = (k + 63) / 64;
  const int splits = choose_splits(tiles, kblocks, num_sms());
  GemmShape sh = make_shape(rows_w, rows_w2, rows_x, k, bn, splits);
  // Stream-K over (m-tile, k-block) when it beats the best even split: every
  // CTA streams an equal share of the weights, and a tile shared by several
  // CTAs gets one partial slab per CTA (the tile's last CTA zeroes the slabs
  // its tile does not use, so the reductions still sum `splits` slabs).
  if (sh.tiles_n == 1) {
    const StreamK sk = plan_stream_k(sh.tiles_m, kblocks, num_sms());
    const long long t_split = (((long long)sh.units + num_sms() - 1) / num_sms()) *
                              (sh.kb_per_split + L3_SPLIT_UNIT_COST);
    if (sk.ok && sk.cost < t_split) {
      sh.sk_per = sk.per;
      sh.units = sk.ctas;
      sh.splits = sk.slabs;
    }
  }
  return sh;
}

int swapped_partial_gemm(const void* w, int rows_w, const void* w_second, int rows_w2, int out_offset2,
                         const void* x, int rows_x, int k, float* P, int ldo, int* splits_out,
                         cudaStream_t st) {
  CUtensorMap ma, ma2, mb;
  const int bn = rows_x <= 16 ? 16 : rows_x <= 32 ? 32 : rows_x <= 64 ? 64 : rows_x <= 128 ? 128 : 256;
  L3_TRY(make_map(&ma, w, rows_w, k, 128));
  if (w_second) L3_TRY(make_map(&ma2, w_second, rows_w2, k, 128)); else ma2 = ma;
  L3_TRY(make_map(&mb, x, rows_x, k, bn));
  GemmShape sh = plan_swapped(rows_w, w_second ? rows_w2 : 0, rows_x, k, bn);
  EpiParams ep = empty_epi();
  ep.out = P;
  ep.ldo = ldo;
  ep.split_stride = (long long)rows_x * ldo;
  ep.out_row_offset2 = out_offset2;
  *splits_out = sh.splits;
  switch (bn) {
    case 16: return launch_gemm<16, 8, EPI_PARTIAL, false>(LLAMA3_KERNEL_DECODE_GEMM, ma, ma2, mb, mb, sh, ep, st);
    case 32: return launch_gemm<32, 8, EPI_PARTIAL, false>(LLAMA3_KERNEL_DECODE_GEMM, ma, ma2, mb, mb, sh, ep, st);
    case 64: return launch_gemm<64, 6, EPI_PARTIAL, false>(LLAMA3_KERNEL_DECODE_GEMM, ma, ma2, mb, mb, sh, ep, st);
    case 128: return launch_gemm<128, 5, EPI_PARTIAL, false>(LLAMA3_KERNEL_DECODE_GEMM, ma, ma2, mb, mb, sh, ep, st);
    default: return launch_gemm<256, 4, EPI_PARTIAL, false>(LLAMA3_KERNEL_DECODE_GEMM, ma, ma2, mb, mb, sh, ep, st);
  }
}


constexpr int kPrefillBN = 256;

// ---------------------------------------------------------------------------
// SIMT helpers (templated on element type)
// ---------------------------------------------------------------------------
template <typename T>
int simt_gemm(int kind, const void* A, const void* B, float* C, int M, int N, int K, int ldc, cudaStream_t st) {
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  L3_LAUNCH(kind, st, launch_k((gemm_simt_kernel<T>), grid, 256, 0, st, (const T*)A, (const T*)B, C, M, N, K, ldc));
  return launch_check();
}

unsigned blocks_for(long long n, int threads) { return (unsigned)((n + threads - 1) / threads); }

template <typename T>
int run_rmsnorm(const llama3_config* c, const void* x, long long row_stride, const void* w, void* y, int rows,
                cudaStream_t st) {
  L3_LAUNCH(LLAMA3_KERNEL_NORM, st, launch_k((rmsnorm_kernel<T>), rows, 256, 0, st, (const T*)x, row_stride, (const T*)w, (T*)y, c->dim, c->norm_eps));
  return launch_check();
}
template <int CPL>
int run_rmsnorm_warp(const llama3_config* c, const void* x, long long row_stride, const void* w, void* y, int rows,
                     cudaStream_t st) {
  L3_LAUNCH(LLAMA3_KERNEL_NORM, st,
            launch_k((rmsnorm_bf16_warp_kernel<CPL>), (rows + 3) / 4, 128, 0, st, (const bf16*)x, row_stride,
                     (const bf16*)w, (bf16*)y, rows, c->dim, c->norm_eps));
  return launch_check();
}

bool rmsnorm_rows_kernel_ok(const llama3_config* c, long long row_stride, int rows) {
  return c->dtype == LLAMA3_DTYPE_BF16 && c->dim % 8 == 0 && (row_stride * 2) % 16 == 0 && g_kernel_path == 0 &&
         rows <= 512 && c->dim / 8 <= 1024;
}

int rmsnorm_any(const llama3_config* c, const void* x, long long row_stride, const void* w, void* y, int rows,
                cudaStream_t st) {
  if (rmsnorm_rows_kernel_ok(c, row_stride, rows)) {
    // few rows (decode, LM head): one CTA per row spreads them over the SMs
    const int threads = (c->dim / 8 + 31) / 32 * 32;
    L3_LAUNCH(LLAMA3_KERNEL_NORM, st,
              launch_k(rmsnorm_bf16_row_kernel, rows, threads, 0, st, (const bf16*)x, row_stride, (const bf16*)w,
                       (bf16*)y, c->dim, c->norm_eps));
    return launch_check();
  }
  if (c->dtype == LLAMA3_DTYPE_F32) return run_rmsnorm<float>(c, x, row_stride, w, y, rows, st);
  // bf16: the warp-per-row kernel when rows are 16-byte aligned and fit its registers
  const int chunks = c->dim / 8;
  if (c->dim % 8 == 0 && (row_stride * 2) % 16 == 0 && g_kernel_path == 0) {
    if (chunks <= 32) return run_rmsnorm_warp<1>(c, x, row_stride, w, y, rows, st);
    if (chunks <= 64) return run_rmsnorm_warp<2>(c, x, row_stride, w, y, rows, st);
    if (chunks <= 128) return run_rmsnorm_warp<4>(c, x, row_stride, w, y, rows, st);
    if (chunks <= 256) return run_rmsnorm_warp<8>(c, x, row_stride, w, y, rows, st);
    if (chunks <= 512) return run_rmsnorm_warp<16>(c, x, row_stride, w, y, rows, st);
    if (chunks <= 1024) return run_rmsnorm_warp<32>(c, x, row_stride, w, y, rows, st);
  }
  return run_rmsnorm<bf16>(c, x, row_stride, w, y, rows, st);
}

template <typename T>
int run_attention_simt(const llama3_config* c, const void* q, const void* kc, const void* vc, int cap, int B,
                       int S, int P, void* out, const int32_t* doc_start, cudaStream_t st,
                       const int32_t* positions = nullptr) {
  const long long warps = (long long)B * S * c->n_heads;
  const float scale = (float)(1.0 / sqrt((double)c->head_dim));
  L3_LAUNCH(LLAMA3_KERNEL_ATTENTION, st, launch_k((attention_simt_kernel<T>), blocks_for(warps * 32, 256), 256, 0, st, 
      (const T*)q, (const T*)kc, (const T*)vc, (T*)out, B, S, P, c->n_heads, c->n_kv_heads, c->head_dim, cap,
      scale, doc_start, positions, P));
  return launch_check();
}

// Decode attention schedule: the segs x tiles key tiles, laid end to end, cut
// into equal runs of *per tiles, one per CTA (*grid of them, at most sms).
// *slots = 2 x the most runs one segment meets (two records per piece); the
// run length grows until that fits the workspace's kMaxKvSplits records.
bool plan_decode_runs(int segs, int tiles, int sms, int* per, int* slots, int* grid) {
  const long long total = (long long)segs * tiles;
  if (total <= 0 || sms <= 0) return false;
  long long p = (total + sms - 1) / sms;
  for (;; ++p) {
    int most = 1;
    for (long long s = 0; s < segs; ++s)
      most = std::max(most, (int)((s * tiles + tiles - 1) / p - (s * tiles) / p + 1));
    if (2 * most <= kMaxKvSplits) {
      *per = (int)p;
      *slots = 2 * most;
      *grid = (int)((total + p - 1) / p);
      return true;
    }
    if (p >= tiles) return false;
  }
}

// Tensor-core decode attention: TMA-streamed K/V tiles, two tcgen05 MMAs per tile.
template <int HD, int NREP>
int run_decode_attention_tc_t(const llama3_config* c, const void* q, const void* kc, const void* vc, int cap,
                              int B, int n_keys, void* out, float* part, cudaStream_t st,
                              const int32_t* positions) {
  using Cfg = DecodeTcCfg<HD>;
  const int KV = c->n_kv_heads, H = c->n_heads;
  const long long e = 2;
  CUtensorMap mq, mk, mv;
  L3_TRY(make_map(&mq, q, (long long)B * H, HD, 16));
  L3_TRY(make_map_4d(&mk, kc, HD, KV, n_keys, B, HD * e, (long long)KV * HD * e, (long long)cap * KV * HD * e));
  L3_TRY(make_map_4d(&mv, vc, HD, KV, n_keys, B, HD * e, (long long)KV * HD * e, (long long)cap * KV * HD * e));
  DecodeShape ds;
  ds.B = B; ds.H = H; ds.KV = KV; ds.nrep = H / KV; ds.n_keys = n_keys;
  ds.tiles = (n_keys + 127) / 128;
  int grid = 0;
  if (!plan_decode_runs(B * KV, ds.tiles, num_sms(), &ds.per, &ds.slots, &grid)) return LLAMA3_ERR_UNSUPPORTED;
  ds.scale_log2 = (float)(1.4426950408889634 / sqrt((double)HD));
  ds.positions = positions;
  auto kern = decode_attention_tc_kernel<HD, NREP>;
  int dev = 0;
  L3_TRY(current_device(&dev));
  static bool attr_done[kMaxDevices];
  if (!attr_done[dev]) {
    L3_CUDA(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES));
    attr_done[dev] = true;
  }
  L3_LAUNCH(LLAMA3_KERNEL_DECODE_ATTENTION, st,
            launch_k(kern, grid, 384, Cfg::SMEM_BYTES, st, mq, mk, mv, part, ds, wait_ns()));
  L3_TRY(launch_check());
  L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st,
            launch_k((decode_attention_combine_kernel<HD>), B * H, 128, 0, st, part, (bf16*)out, ds.slots, H,
                     ds.nrep, ds.tiles, ds.per));
  return launch_check();
}

template <int HD>
int run_decode_attention_tc_hd(const llama3_config* c, const void* q, const void* kc, const void* vc, int cap,
                               int B, int n_keys, void* out, float* part, cudaStream_t st,
                               const int32_t* positions) {
  const int r = c->n_heads / c->n_kv_heads;
  if (r <= 1) return run_decode_attention_tc_t<HD, 1>(c, q, kc, vc, cap, B, n_keys, out, part, st, positions);
  if (r <= 2) return run_decode_attention_tc_t<HD, 2>(c, q, kc, vc, cap, B, n_keys, out, part, st, positions);
  if (r <= 4) return run_decode_attention_tc_t<HD, 4>(c, q, kc, vc, cap, B, n_keys, out, part, st, positions);
  if (r <= 8) return run_decode_attention_tc_t<HD, 8>(c, q, kc, vc, cap, B, n_keys, out, part, st, positions);
  if (r <= 16) return run_decode_attention_tc_t<HD, 16>(c, q, kc, vc, cap, B, n_keys, out, part, st, positions);
  return LLAMA3_ERR_UNSUPPORTED;
}

bool decode_attention_tc_supported(const llama3_config* c) {
  return use_tc(c) && (c->head_dim == 64 || c->head_dim == 96 || c->head_dim == 128) &&
         c->n_heads / c->n_kv_heads <= 16;
}

// positions (device [B], with S == 1 and P = their upper bound): every
// sequence's token at its own position (ragged decode).
int attention_dispatch(const llama3_config* c, const void* q, const void* kc, const void* vc, int cap, int B,
                       int S, int P, void* out, float* part, cudaStream_t st, const int32_t* doc_start = nullptr,
                       const int32_t* positions = nullptr) {
  if (positions) {
    if (S != 1 || doc_start) return LLAMA3_ERR_ARG;
    if (!decode_attention_tc_supported(c))
      return c->dtype == LLAMA3_DTYPE_F32
                 ? run_attention_simt<float>(c, q, kc, vc, cap, B, 1, P, out, nullptr, st, positions)
                 : run_attention_simt<bf16>(c, q, kc, vc, cap, B, 1, P, out, nullptr, st, positions);
  }
  if (S == 1 && !doc_start && decode_attention_tc_supported(c)) {
    switch (c->head_dim) {
      case 64: return run_decode_attention_tc_hd<64>(c, q, kc, vc, cap, B, P + 1, out, part, st, positions);
      case 96: return run_decode_attention_tc_hd<96>(c, q, kc, vc, cap, B, P + 1, out, part, st, positions);
      default: return run_decode_attention_tc_hd<128>(c, q, kc, vc, cap, B, P + 1, out, part, st, positions);
    }
  }
  if (use_tc(c) && flash_attention_supported(c->head_dim, c->n_heads, c->n_kv_heads))
    return run_flash_attention(c->head_dim, c->n_heads, c->n_kv_heads, q, kc, vc, cap, B, S, P, out, doc_start,
                               num_sms(), wait_ns(), st);
  return c->dtype == LLAMA3_DTYPE_F32 ? run_attention_simt<float>(c, q, kc, vc, cap, B, S, P, out, doc_start, st)
                                      : run_attention_simt<bf16>(c, q, kc, vc, cap, B, S, P, out, doc_start, st);
}

// ---------------------------------------------------------------------------
// Layer: SIMT path (any dtype)
// ---------------------------------------------------------------------------
template <typename T>
int layer_simt(const llama3_config* c, const llama3_layer_weights* w, const float* rope, void* x, void* kc,
               void* vc, int cap, int B, int S, int P, const Workspace& L, void* ws, cudaStream_t st,
               const int32_t* doc_start = nullptr, const int32_t* positions = nullptr) {
  const int M = B * S, D = c->dim, H = c->n_heads, KV = c->n_kv_heads, hd = c->head_dim, F = c->ffn_hidden;
  const int nqkv = (H + 2 * KV) * hd;
  T* xn = ws_at<T>(ws, L.xn);
  T* q = ws_at<T>(ws, L.q);
  T* o = ws_at<T>(ws, L.o);
  T* g = ws_at<T>(ws, L.g);
  float* Pp = ws_at<float>(ws, L.part);
  float* Ap = ws_at<float>(ws, L.attn_part);
  L3_TRY(run_rmsnorm<T>(c, x, D, w->attention_norm, xn, M, st));
  L3_TRY(simt_gemm<T>(LLAMA3_KERNEL_GEMM_QKV, xn, w->wqkv, Pp, M, nqkv, D, nqkv, st));
  L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((epi_qkv_rope_kernel<T>), blocks_for((long long)M * nqkv / 4, 256), 256, 0, st, 
      Pp, 1, 0, M, S, P, H, KV, hd, rope, q, (T*)kc, (T*)vc, cap, positions, P));
  L3_TRY(launch_check());
  L3_TRY(attention_dispatch(c, q, kc, vc, cap, B, S, P, o, Ap, st, doc_start, positions));
  L3_TRY(simt_gemm<T>(LLAMA3_KERNEL_GEMM_WO, o, w->wo, Pp, M, D, H * hd, D, st));
  L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((epi_residual_kernel<T>), blocks_for((long long)M * D / 4, 256), 256, 0, st, Pp, 1, 0, D, (const T*)x, (T*)x, M, D));
  L3_TRY(launch_check());
  L3_TRY(run_rmsnorm<T>(c, x, D, w->ffn_norm, xn, M, st));
  L3_TRY(simt_gemm<T>(LLAMA3_KERNEL_GEMM_W13, xn, w->w1, Pp, M, F, D, 2 * F, st));
  L3_TRY(simt_gemm<T>(LLAMA3_KERNEL_GEMM_W13, xn, w->w3, Pp + F, M, F, D, 2 * F, st));
  L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((epi_swiglu_kernel<T>), blocks_for((long long)M * F / 4, 256), 256, 0, st, Pp, 1, 0, g, M, F));
  L3_TRY(launch_check());
  L3_TRY(simt_gemm<T>(LLAMA3_KERNEL_GEMM_W2, g, w->w2, Pp, M, D, F, D, st));
  L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((epi_residual_kernel<T>), blocks_for((long long)M * D / 4, 256), 256, 0, st, Pp, 1, 0, D, (const T*)x, (T*)x, M, D));
  return launch_check();
}

// ---------------------------------------------------------------------------
// Layer: tcgen05 prefill path (bf16)
// ---------------------------------------------------------------------------
int layer_tc_prefill(const llama3_config* c, const llama3_layer_weights* w, const float* rope, void* x, void* kc,
                     void* vc, int cap, int B, int S, int P, const Workspace& L, void* ws, cudaStream_t st,
                     const int32_t* doc_start = nullptr) {
  const int M = B * S, D = c->dim, H = c->n_heads, KV = c->n_kv_heads, hd = c->head_dim, F = c->ffn_hidden;
  const int nqkv = (H + 2 * KV) * hd;
  bf16* xn = ws_at<bf16>(ws, L.xn);
  bf16* q = ws_at<bf16>(ws, L.q);
  bf16* o = ws_at<bf16>(ws, L.o);
  bf16* g = ws_at<bf16>(ws, L.g);
  float* Ap = ws_at<float>(ws, L.attn_part);
  CUtensorMap mxn, mo, mg, mwqkv, mwo, mw1, mw3, mw2;
  // CTA-pair GEMMs take each weight tile in halves, one per CTA (box rows BN / 2)
  const bool pair = use_pair_gemm(M);
  const int bb = pair ? kPrefillBN / 2 : kPrefillBN;
  const int bd = pair ? 64 : 128;
  L3_TRY(make_map(&mxn, xn, M, D, 128));
  L3_TRY(make_map(&mo, o, M, H * hd, 128));
  L3_TRY(make_map(&mg, g, M, F, 128));
  L3_TRY(make_map(&mwqkv, w->wqkv, nqkv, D, bb));
  L3_TRY(make_map(&mwo, w->wo, D, H * hd, bb));
  L3_TRY(make_map(&mw1, w->w1, F, D, bd));
  L3_TRY(make_map(&mw3, w->w3, F, D, bd));
  L3_TRY(make_map(&mw2, w->w2, D, F, bb));

  // attention half
  L3_TRY(rmsnorm_any(c, x, D, w->attention_norm, xn, M, st));
  {
    EpiParams ep = empty_epi();
    ep.seq = S; ep.start_pos = P; ep.n_heads = H; ep.n_kv = KV; ep.head_dim = hd; ep.cache_cap = cap;
    ep.rope = rope; ep.q_out = q; ep.k_cache = kc; ep.v_cache = vc;
    if (pair)
      L3_TRY((launch_gemm_pair<kPrefillBN, 6, EPI_QKV_ROPE, false>(
          LLAMA3_KERNEL_GEMM_QKV, mxn, mwqkv, mwqkv, make_shape_pair(M, nqkv, D, kPrefillBN), ep, st)));
    else
      L3_TRY((launch_gemm<kPrefillBN, 4, EPI_QKV_ROPE, false>(LLAMA3_KERNEL_GEMM_QKV, mxn, mxn, mwqkv, mwqkv,
                                                               make_shape(M, 0, nqkv, D, kPrefillBN, 1), ep, st)));
  }
  L3_TRY(attention_dispatch(c, q, kc, vc, cap, B, S, P, o, Ap, st, doc_start));
  {
    EpiParams ep = empty_epi();
    ep.out = x; ep.res = x; ep.ldo = D;
    if (pair)
      L3_TRY((launch_gemm_pair<kPrefillBN, 6, EPI_RESIDUAL, false>(
          LLAMA3_KERNEL_GEMM_WO, mo, mwo, mwo, make_shape_pair(M, D, H * hd, kPrefillBN), ep, st)));
    else
      L3_TRY((launch_gemm<kPrefillBN, 4, EPI_RESIDUAL, false>(LLAMA3_KERNEL_GEMM_WO, mo, mo, mwo, mwo,
                                                               make_shape(M, 0, D, H * hd, kPrefillBN, 1), ep, st)));
  }
  // FFN half
  L3_TRY(rmsnorm_any(c, x, D, w->ffn_norm, xn, M, st));
  {
    EpiParams ep = empty_epi();
    ep.out = g; ep.ldo = F;
    if (pair)
      L3_TRY((launch_gemm_pair<128, 6, EPI_SWIGLU, true>(LLAMA3_KERNEL_GEMM_W13, mxn, mw1, mw3,
                                                          make_shape_pair(M, F, D, 128), ep, st)));
    else
      L3_TRY((launch_gemm<128, 4, EPI_SWIGLU, true>(LLAMA3_KERNEL_GEMM_W13, mxn, mxn, mw1, mw3,
                                                     make_shape(M, 0, F, D, 128, 1), ep, st)));
  }
  {
    EpiParams ep = empty_epi();
    ep.out = x; ep.res = x; ep.ldo = D;
    if (pair)
      L3_TRY((launch_gemm_pair<kPrefillBN, 6, EPI_RESIDUAL, false>(
          LLAMA3_KERNEL_GEMM_W2, mg, mw2, mw2, make_shape_pair(M, D, F, kPrefillBN), ep, st)));
    else
      L3_TRY((launch_gemm<kPrefillBN, 4, EPI_RESIDUAL, false>(LLAMA3_KERNEL_GEMM_W2, mg, mg, mw2, mw2,
                                                               make_shape(M, 0, D, F, kPrefillBN, 1), ep, st)));
  }
  return LLAMA3_OK;
}

// ---------------------------------------------------------------------------
// Layer: tcgen05 decode path (bf16, few tokens): weight-streaming split-K
// GEMMs + SIMT epilogues over the fp32 partials.
// ---------------------------------------------------------------------------
// next_norm: also leave RMSNorm(x_out, next_norm) in the workspace's normalised-
// input buffer for the next block; input_normalised: that buffer already holds
// this block's RMSNorm(x, attention_norm) (left by the previous block).
int layer_tc_decode(const llama3_config* c, const llama3_layer_weights* w, const float* rope, void* x, void* kc,
                    void* vc, int cap, int B, int P, const Workspace& L, void* ws, cudaStream_t st,
                    const int32_t* positions = nullptr, const void* next_norm = nullptr,
                    bool input_normalised = false) {
  const int M = B, D = c->dim, H = c->n_heads, KV = c->n_kv_heads, hd = c->head_dim, F = c->ffn_hidden;
  const int nqkv = (H + 2 * KV) * hd;
  bf16* xn = ws_at<bf16>(ws, L.xn);
  bf16* q = ws_at<bf16>(ws, L.q);
  bf16* o = ws_at<bf16>(ws, L.o);
  bf16* g = ws_at<bf16>(ws, L.g);
  float* Pp = ws_at<float>(ws, L.part);
  float* Ap = ws_at<float>(ws, L.attn_part);
  int splits = 1;
  if (!input_normalised) L3_TRY(rmsnorm_any(c, x, D, w->attention_norm, xn, M, st));
  L3_TRY(swapped_partial_gemm(w->wqkv, nqkv, nullptr, 0, 0, xn, M, D, Pp, nqkv, &splits, st));
  L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((epi_qkv_rope_kernel<bf16>), blocks_for((long long)M * nqkv / 4, 256), 256, 0, st,
      Pp, splits, (long long)M * nqkv, M, 1, P, H, KV, hd, rope, q, (bf16*)kc, (bf16*)vc, cap, positions, P));
  L3_TRY(launch_check());
  L3_TRY(attention_dispatch(c, q, kc, vc, cap, B, 1, P, o, Ap, st, nullptr, positions));
  // x += the split sums (row-wise), then xn = RMSNorm(x, norm_w), in one pass
  // over each row where the row fits one CTA
  auto residual_then_norm = [&](const void* norm_w) -> int {
    if (D <= 4 * 4 * 1024) {
      const int G = (D + 4095) / 4096;
      const long long sstride = (long long)M * D;
      if (G <= 1)
        L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((epi_residual_rmsnorm_kernel<1>), M, 1024, 0, st, Pp, splits,
                                                          sstride, (bf16*)x, (const bf16*)norm_w, xn, D, c->norm_eps));
      else if (G <= 2)
        L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((epi_residual_rmsnorm_kernel<2>), M, 1024, 0, st, Pp, splits,
                                                          sstride, (bf16*)x, (const bf16*)norm_w, xn, D, c->norm_eps));
      else
        L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((epi_residual_rmsnorm_kernel<4>), M, 1024, 0, st, Pp, splits,
                                                          sstride, (bf16*)x, (const bf16*)norm_w, xn, D, c->norm_eps));
      return launch_check();
    }
    L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((epi_residual_kernel<bf16>), blocks_for((long long)M * D / 4, 256),
                                                      256, 0, st, Pp, splits, (long long)M * D, D, (const bf16*)x,
                                                      (bf16*)x, M, D));
    L3_TRY(launch_check());
    return rmsnorm_any(c, x, D, norm_w, xn, M, st);
  };
  L3_TRY(swapped_partial_gemm(w->wo, D, nullptr, 0, 0, o, M, H * hd, Pp, D, &splits, st));
  // h = x + o Wo^T and hn = RMSNorm(h)
  L3_TRY(residual_then_norm(w->ffn_norm));
  L3_TRY(swapped_partial_gemm(w->w1, F, w->w3, F, F, xn, M, D, Pp, 2 * F, &splits, st));
  L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((epi_swiglu_kernel<bf16>), blocks_for((long long)M * F / 4, 256), 256, 0, st, Pp, splits, (long long)M * 2 * F, g,
                                                                                M, F));
  L3_TRY(launch_check());
  L3_TRY(swapped_partial_gemm(w->w2, D, nullptr, 0, 0, g, M, F, Pp, D, &splits, st));
  // out = h + g W2^T, and with next_norm the next block's normalised input
  if (next_norm) return residual_then_norm(next_norm);
  L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((epi_residual_kernel<bf16>), blocks_for((long long)M * D / 4, 256), 256, 0, st,
      Pp, splits, (long long)M * D, D, (const bf16*)x, (bf16*)x, M, D));
  return launch_check();
}

int check_layer_args(const llama3_config* c, const llama3_layer_weights* w, const float* rope, int rope_len,
                     const void* x, const void* kc, const void* vc, int cap, int B, int S, int P, const void* ws,
                     size_t ws_bytes, Workspace* L) {
  L3_TRY(check_config(c));
  if (!w || !rope || !x || !kc || !vc) return LLAMA3_ERR_ARG;
  if (B < 1 || S < 1 || P < 0 || cap < 1) return LLAMA3_ERR_ARG;
  if ((long long)P + S > cap) return LLAMA3_ERR_ARG;
  if ((long long)P + S > rope_len) return LLAMA3_ERR_ARG;
  const void* ptrs[] = {w->attention_norm, w->wqkv, w->wo, w->ffn_norm, w->w1, w->w2, w->w3, rope, x, kc, vc};
  for (const void* p : ptrs) {
    if (!p) return LLAMA3_ERR_ARG;
    if (!aligned16(p)) return LLAMA3_ERR_ALIGN;
  }
  *L = layout(c, B, S, 1);
  if (!ws || ws_bytes < L->total) return LLAMA3_ERR_WORKSPACE;
  if (!aligned16(ws)) return LLAMA3_ERR_ALIGN;
  return LLAMA3_OK;
}

// Argument checks shared by both LM-head entry points.
int check_lm_head_args(const llama3_config* cfg, const void* norm_w, const void* w_out, const void* h, int rows,
                       long long row_stride, const int32_t* ids_out, const float* logits_out) {
  L3_TRY(check_config(cfg));
  if (!norm_w || !w_out || !h || !ids_out || rows < 1 || cfg->vocab < 1 || row_stride < cfg->dim)
    return LLAMA3_ERR_ARG;
  if (!aligned16(norm_w) || !aligned16(w_out) || !aligned16(h) || !aligned16(ids_out) ||
      (logits_out && !aligned16(logits_out)))
    return LLAMA3_ERR_ALIGN;
  if ((row_stride * (long long)esize(cfg)) % 16) return LLAMA3_ERR_ALIGN;
  return LLAMA3_OK;
}

// Final RMSNorm -> logits -> argmax of `rows` rows, with its scratch where the
// caller of this helper chose: hn (rows x dim elements, 16-byte aligned) for
// the normalised rows and keys (rows 64-bit words) for the packed per-row
// maxima.  The keys are re-initialised here on every call.
int lm_head_run(const llama3_config* cfg, const void* norm_w, const void* w_out, const void* h, int rows,
                long long row_stride, int32_t* ids_out, float* logits_out, void* hn, unsigned long long* keys,
                cudaStream_t st) {
  const int V = cfg->vocab, D = cfg->dim;
  L3_TRY(rmsnorm_any(cfg, h, row_stride, norm_w, hn, rows, st));
  L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st,
            launch_k((argmax_init_kernel), blocks_for(rows, 256), 256, 0, st, keys, rows));
  L3_TRY(launch_check());
  if (use_tc(cfg)) {
    const int bn = rows <= 16 ? 16 : rows <= 32 ? 32 : rows <= 64 ? 64 : rows <= 128 ? 128 : 256;
    CUtensorMap ma, mb;
    L3_TRY(make_map(&ma, w_out, V, D, 128));
    L3_TRY(make_map(&mb, hn, rows, D, bn));
    GemmShape sh = make_shape(V, 0, rows, D, bn, 1);
    EpiParams ep = empty_epi();
    ep.logits = logits_out;
    ep.keys = keys;
    switch (bn) {
      case 16: L3_TRY((launch_gemm<16, 8, EPI_ARGMAX, false>(LLAMA3_KERNEL_LM_HEAD, ma, ma, mb, mb, sh, ep, st))); break;
      case 32: L3_TRY((launch_gemm<32, 8, EPI_ARGMAX, false>(LLAMA3_KERNEL_LM_HEAD, ma, ma, mb, mb, sh, ep, st))); break;
      case 64: L3_TRY((launch_gemm<64, 6, EPI_ARGMAX, false>(LLAMA3_KERNEL_LM_HEAD, ma, ma, mb, mb, sh, ep, st))); break;
      case 128: L3_TRY((launch_gemm<128, 5, EPI_ARGMAX, false>(LLAMA3_KERNEL_LM_HEAD, ma, ma, mb, mb, sh, ep, st))); break;
      default: L3_TRY((launch_gemm<256, 4, EPI_ARGMAX, false>(LLAMA3_KERNEL_LM_HEAD, ma, ma, mb, mb, sh, ep, st))); break;
    }
  } else {
    const long long warps = (long long)rows * ((V + 31) / 32);
    if (cfg->dtype == LLAMA3_DTYPE_F32)
      L3_LAUNCH(LLAMA3_KERNEL_LM_HEAD, st,
                launch_k((lm_head_simt_kernel<float>), blocks_for(warps * 32, 256), 256, 0, st, (const float*)hn,
                         (const float*)w_out, logits_out, keys, rows, V, D));
    else
      L3_LAUNCH(LLAMA3_KERNEL_LM_HEAD, st,
                launch_k((lm_head_simt_kernel<bf16>), blocks_for(warps * 32, 256), 256, 0, st, (const bf16*)hn,
                         (const bf16*)w_out, logits_out, keys, rows, V, D));
    L3_TRY(launch_check());
  }
  L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st,
            launch_k((argmax_finalize_kernel), blocks_for(rows, 256), 256, 0, st, keys, ids_out, rows));
  return launch_check();
}

}  // namespace

// ===========================================================================
// C ABI
// ===========================================================================
extern "C" {

const char* llama3_status_string(int s) {
  switch (s) {
    case LLAMA3_OK: return "ok";
    case LLAMA3_ERR_ARG: return "invalid argument";
    case LLAMA3_ERR_ALIGN: return "pointer or stride not 16-byte aligned";
    case LLAMA3_ERR_WORKSPACE: return "workspace missing or too small";
    case LLAMA3_ERR_CUDA: return "CUDA call failed (see llama3_last_cuda_error)";
    case LLAMA3_ERR_TIMEOUT: return "device-side wait timed out";
    case LLAMA3_ERR_TOKEN: return "token id out of range";
    case LLAMA3_ERR_UNSUPPORTED: return "shape not supported by the kernels";
    default: return "unknown status";
  }
}

int llama3_last_cuda_error(void) { return t_last_cuda; }

int llama3_set_launch_timer(int kind, void* const* start_events, void* const* stop_events, int n_pairs) {
  if (n_pairs < 0 || (n_pairs > 0 && (!start_events || !stop_events))) return LLAMA3_ERR_ARG;
  g_timer.kind = n_pairs ? kind : 0;
  g_timer.n = n_pairs;
  g_timer.used = 0;
  g_timer.start.assign(n_pairs, nullptr);
  g_timer.stop.assign(n_pairs, nullptr);
  for (int i = 0; i < n_pairs; ++i) {
    g_timer.start[i] = (cudaEvent_t)start_events[i];
    g_timer.stop[i] = (cudaEvent_t)stop_events[i];
  }
  return LLAMA3_OK;
}

int llama3_launch_timer_used(void) { return g_timer.used; }

unsigned long long llama3_launch_count(void) { return g_launches.load(); }

int llama3_set_kernel_path(int path) {
  int old = g_kernel_path;
  g_kernel_path = (path == 1) ? 1 : 0;
  return old;
}

int llama3_sample_top_p(const float* logits, int rows, long long ld, int vocab, float temperature, float top_p,
                        unsigned long long seed, unsigned long long offset, const int32_t* positions,
                        int32_t* ids_out, llama3_stream_t stream) {
  if (!logits || !ids_out || rows < 1 || vocab < 1 || ld < vocab) return LLAMA3_ERR_ARG;
  if (std::isnan(temperature) || std::isnan(top_p) || top_p < 0.f) return LLAMA3_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(logits) & 3) || (reinterpret_cast<uintptr_t>(ids_out) & 3) ||
      (reinterpret_cast<uintptr_t>(positions) & 3))
    return LLAMA3_ERR_ALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  int dev = 0;
  L3_TRY(current_device(&dev));
  static bool attr_done[kMaxDevices];
  if (!attr_done[dev]) {
    L3_CUDA(cudaFuncSetAttribute(sample_top_p_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSampleSmem));
    attr_done[dev] = true;
  }
  SampleParams sp;
  sp.logits = logits;
  sp.ld = ld;
  sp.V = vocab;
  sp.temperature = temperature;
  sp.top_p = top_p;
  sp.seed = seed;
  sp.offset = offset;
  sp.positions = positions;
  sp.ids = ids_out;
  L3_LAUNCH(LLAMA3_KERNEL_SAMPLE, st, launch_k(sample_top_p_kernel, rows, kSampleThreads, kSampleSmem, st, sp));
  return launch_check();
}

int llama3_gather_rows(const llama3_config* cfg, const void* x, long long row_stride, int n_rows,
                       const int32_t* row_index, int rows, void* out, llama3_stream_t stream) {
  L3_TRY(check_config(cfg));
  if (!x || !row_index || !out || rows < 1 || n_rows < 1 || row_stride < cfg->dim) return LLAMA3_ERR_ARG;
  const long long es = esize(cfg);
  if (!aligned16(x) || !aligned16(out) || (reinterpret_cast<uintptr_t>(row_index) & 3) ||
      (row_stride * es) % 16 || ((long long)cfg->dim * es) % 16)
    return LLAMA3_ERR_ALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st,
            launch_k(gather_rows_kernel, rows, 128, 0, st, (const uint4*)x, row_stride * es / 16, row_index, n_rows,
                     (uint4*)out, (int)((long long)cfg->dim * es / 16)));
  return launch_check();
}

int llama3_generation_advance(int32_t* positions, int32_t* ids, int32_t* history, int32_t* step, int32_t* done,
                              int eos_id, int batch, int history_rows, long long history_stride,
                              llama3_stream_t stream) {
  if (!positions || !ids || !history || !step || batch < 1 || history_rows < 1 || history_stride < batch)
    return LLAMA3_ERR_ARG;
  if (eos_id >= 0 && !done) return LLAMA3_ERR_ARG;
  const uintptr_t any = reinterpret_cast<uintptr_t>(positions) | reinterpret_cast<uintptr_t>(ids) |
                        reinterpret_cast<uintptr_t>(history) | reinterpret_cast<uintptr_t>(step) |
                        reinterpret_cast<uintptr_t>(done);
  if (any & 3) return LLAMA3_ERR_ALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  int32_t* d = eos_id >= 0 ? done : nullptr;
  L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k(generation_advance_kernel, 1, 256, 0, st, positions, ids, history,
                                                    step, d, eos_id, batch, history_rows, history_stride));
  return launch_check();
}

int llama3_set_programmatic_launch(int on) {
  const int old = g_pdl ? 1 : 0;
  g_pdl = on != 0;
  return old;
}

int llama3_set_wait_limit_ms(int ms) {
  int old = g_wait_ms;
  if (ms > 0) g_wait_ms = ms;
  return old;
}

int llama3_set_test_withheld_arrival(int which) {
  const int old = g_withhold;
  g_withhold = (which == 1 || which == 2) ? which : 0;
  return old;
}

int llama3_device_status(int* out) {
  if (!out) return LLAMA3_ERR_ARG;
  int v = 0, zero = 0;
  L3_CUDA(cudaDeviceSynchronize());
  L3_CUDA(cudaMemcpyFromSymbol(&v, g_status, sizeof(int)));
  L3_CUDA(cudaMemcpyToSymbol(g_status, &zero, sizeof(int)));
  *out = v;
  return LLAMA3_OK;
}

int llama3_init_rope_table(float* cos_sin, int head_dim, int max_pos, double theta, llama3_stream_t stream) {
  if (!cos_sin || head_dim < 2 || (head_dim & 1) || max_pos < 1 || !(theta > 1.0)) return LLAMA3_ERR_ARG;
  if (!aligned16(cos_sin)) return LLAMA3_ERR_ALIGN;
  const int half = head_dim / 2;
  const size_t n = (size_t)max_pos * half * 2;
  std::vector<float> host(n);
  for (int m = 0; m < max_pos; ++m) {
    for (int i = 0; i < half; ++i) {
      const double inv = pow(theta, -(2.0 * i) / (double)head_dim);
      const double ang = (double)m * inv;
      host[((size_t)m * half + i) * 2] = (float)cos(ang);
      host[((size_t)m * half + i) * 2 + 1] = (float)sin(ang);
    }
  }
  L3_CUDA(cudaMemcpyAsync(cos_sin, host.data(), n * sizeof(float), cudaMemcpyHostToDevice, (cudaStream_t)stream));
  L3_CUDA(cudaStreamSynchronize((cudaStream_t)stream));
  return LLAMA3_OK;
}

int llama3_workspace_size(const llama3_config* cfg, int batch, int seq, int lm_rows, size_t* bytes) {
  L3_TRY(check_config(cfg));
  if (!bytes || batch < 1 || seq < 1 || lm_rows < 0) return LLAMA3_ERR_ARG;
  *bytes = layout(cfg, batch, seq, lm_rows).total;
  return LLAMA3_OK;
}

int llama3_embed(const llama3_config* cfg, const int32_t* ids, const void* table, void* x, int n_tokens,
                 llama3_stream_t stream) {
  L3_TRY(check_config(cfg));
  if (!ids || !table || !x || n_tokens < 1 || cfg->vocab < 1) return LLAMA3_ERR_ARG;
  if (!aligned16(ids) || !aligned16(table) || !aligned16(x)) return LLAMA3_ERR_ALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  if (cfg->dtype == LLAMA3_DTYPE_F32)
    L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((embed_kernel<float>), n_tokens, 128, 0, st, ids, (const float*)table, (float*)x, cfg->dim, cfg->vocab));
  else
    L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((embed_kernel<bf16>), n_tokens, 128, 0, st, ids, (const bf16*)table, (bf16*)x, cfg->dim, cfg->vocab));
  return launch_check();
}

int llama3_rmsnorm(const llama3_config* cfg, const void* x, long long row_stride, const void* w, void* y, int rows,
                   llama3_stream_t stream) {
  L3_TRY(check_config(cfg));
  if (!x || !w || !y || rows < 1 || row_stride < cfg->dim) return LLAMA3_ERR_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y)) return LLAMA3_ERR_ALIGN;
  return rmsnorm_any(cfg, x, row_stride, w, y, rows, (cudaStream_t)stream);
}

int llama3_linear(const llama3_config* cfg, const void* x, const void* w, const void* residual, void* y, int m,
                  int n, int k, void* ws, size_t ws_bytes, llama3_stream_t stream) {
  L3_TRY(check_config(cfg));
  if (!x || !w || !y || m < 1 || n < 1 || k < 1) return LLAMA3_ERR_ARG;
  if (!aligned16(x) || !aligned16(w) || !aligned16(y) || (residual && !aligned16(residual)))
    return LLAMA3_ERR_ALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  if (use_tc(cfg)) {
    if (k % 8 || n % 8) return LLAMA3_ERR_ALIGN;
    CUtensorMap ma, mb;
    EpiParams ep = empty_epi();
    ep.out = y; ep.res = residual; ep.ldo = n;
    L3_TRY(make_map(&ma, x, m, k, 128));
    if (use_pair_gemm(m)) {
      L3_TRY(make_map(&mb, w, n, k, kPrefillBN / 2));
      const GemmShape sh = make_shape_pair(m, n, k, kPrefillBN);
      if (residual) return launch_gemm_pair<kPrefillBN, 6, EPI_RESIDUAL, false>(LLAMA3_KERNEL_GEMM_WO, ma, mb, mb, sh, ep, st);
      return launch_gemm_pair<kPrefillBN, 6, EPI_STORE, false>(LLAMA3_KERNEL_GEMM_WO, ma, mb, mb, sh, ep, st);
    }
    L3_TRY(make_map(&mb, w, n, k, kPrefillBN));
    GemmShape sh = make_shape(m, 0, n, k, kPrefillBN, 1);
    if (residual) return launch_gemm<kPrefillBN, 4, EPI_RESIDUAL, false>(LLAMA3_KERNEL_GEMM_WO, ma, ma, mb, mb, sh, ep, st);
    return launch_gemm<kPrefillBN, 4, EPI_STORE, false>(LLAMA3_KERNEL_GEMM_WO, ma, ma, mb, mb, sh, ep, st);
  }
  if (n % 4) return LLAMA3_ERR_ALIGN;
  const size_t need = (size_t)m * n * 4;
  if (!ws || ws_bytes < need) return LLAMA3_ERR_WORKSPACE;
  float* C = (float*)ws;
  if (cfg->dtype == LLAMA3_DTYPE_F32) {
    L3_TRY(simt_gemm<float>(LLAMA3_KERNEL_GEMM_WO, x, w, C, m, n, k, n, st));
    L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((epi_residual_kernel<float>), blocks_for(((long long)m * n + 3) / 4, 256), 256, 0, st, C, 1, 0, n, (const float*)residual,
                                                                                  (float*)y, m, n));
  } else {
    L3_TRY(simt_gemm<bf16>(LLAMA3_KERNEL_GEMM_WO, x, w, C, m, n, k, n, st));
    L3_LAUNCH(LLAMA3_KERNEL_ELEMENTWISE, st, launch_k((epi_residual_kernel<bf16>), blocks_for(((long long)m * n + 3) / 4, 256), 256, 0, st, C, 1, 0, n, (const bf16*)residual,
                                                                                 (bf16*)y, m, n));
  }
  return launch_check();
}

int llama3_attention(const llama3_config* cfg, const void* q, const void* k_cache, const void* v_cache,
                     int cache_cap, int batch, int seq, int start_pos, void* out, void* ws, size_t ws_bytes,
                     llama3_stream_t stream) {
  L3_TRY(check_config(cfg));
  if (!q || !k_cache || !v_cache || !out || batch < 1 || seq < 1 || start_pos < 0) return LLAMA3_ERR_ARG;
  if ((long long)start_pos + seq > cache_cap) return LLAMA3_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out)) return LLAMA3_ERR_ALIGN;
  Workspace L = layout(cfg, batch, seq, 1);
  if (!ws || ws_bytes < L.total) return LLAMA3_ERR_WORKSPACE;
  return attention_dispatch(cfg, q, k_cache, v_cache, cache_cap, batch, seq, start_pos, out,
                            ws_at<float>(ws, L.attn_part), (cudaStream_t)stream);
}

int llama3_layer_forward(const llama3_config* cfg, const llama3_layer_weights* w, const float* rope, int rope_len,
                         void* x, void* k_cache, void* v_cache, int cache_cap, int batch, int seq, int start_pos,
                         void* ws, size_t ws_bytes, llama3_stream_t stream) {
  Workspace L;
  L3_TRY(check_layer_args(cfg, w, rope, rope_len, x, k_cache, v_cache, cache_cap, batch, seq, start_pos, ws,
                          ws_bytes, &L));
  cudaStream_t st = (cudaStream_t)stream;
  if (use_tc(cfg))
    return layer_tc_prefill(cfg, w, rope, x, k_cache, v_cache, cache_cap, batch, seq, start_pos, L, ws, st);
  if (cfg->dtype == LLAMA3_DTYPE_F32)
    return layer_simt<float>(cfg, w, rope, x, k_cache, v_cache, cache_cap, batch, seq, start_pos, L, ws, st);
  return layer_simt<bf16>(cfg, w, rope, x, k_cache, v_cache, cache_cap, batch, seq, start_pos, L, ws, st);
}

int llama3_layer_decode(const llama3_config* cfg, const llama3_layer_weights* w, const float* rope, int rope_len,
                        void* x, void* k_cache, void* v_cache, int cache_cap, int batch, int start_pos, void* ws,
                        size_t ws_bytes, llama3_stream_t stream) {
  Workspace L;
  L3_TRY(check_layer_args(cfg, w, rope, rope_len, x, k_cache, v_cache, cache_cap, batch, 1, start_pos, ws,
                          ws_bytes, &L));
  cudaStream_t st = (cudaStream_t)stream;
  if (use_tc(cfg)) {
    if (batch <= 256)
      return layer_tc_decode(cfg, w, rope, x, k_cache, v_cache, cache_cap, batch, start_pos, L, ws, st);
    return layer_tc_prefill(cfg, w, rope, x, k_cache, v_cache, cache_cap, batch, 1, start_pos, L, ws, st);
  }
  if (cfg->dtype == LLAMA3_DTYPE_F32)
    return layer_simt<float>(cfg, w, rope, x, k_cache, v_cache, cache_cap, batch, 1, start_pos, L, ws, st);
  return layer_simt<bf16>(cfg, w, rope, x, k_cache, v_cache, cache_cap, batch, 1, start_pos, L, ws, st);
}

int llama3_layer_decode_ragged(const llama3_config* cfg, const llama3_layer_weights* w, const float* rope,
                               int rope_len, void* x, void* k_cache, void* v_cache, int cache_cap, int batch,
                               const int32_t* positions, int max_position, void* ws, size_t ws_bytes,
                               llama3_stream_t stream) {
  if (!positions) return LLAMA3_ERR_ARG;
  if (reinterpret_cast<uintptr_t>(positions) & 3) return LLAMA3_ERR_ALIGN;
  Workspace L;
  L3_TRY(check_layer_args(cfg, w, rope, rope_len, x, k_cache, v_cache, cache_cap, batch, 1, max_position, ws,
                          ws_bytes, &L));
  cudaStream_t st = (cudaStream_t)stream;
  if (use_tc(cfg))
    return layer_tc_decode(cfg, w, rope, x, k_cache, v_cache, cache_cap, batch, max_position, L, ws, st, positions);
  if (cfg->dtype == LLAMA3_DTYPE_F32)
    return layer_simt<float>(cfg, w, rope, x, k_cache, v_cache, cache_cap, batch, 1, max_position, L, ws, st,
                             nullptr, positions);
  return layer_simt<bf16>(cfg, w, rope, x, k_cache, v_cache, cache_cap, batch, 1, max_position, L, ws, st,
                          nullptr, positions);
}

int llama3_layer_decode_chained(const llama3_config* cfg, const llama3_layer_weights* w, const float* rope,
                                int rope_len, void* x, void* k_cache, void* v_cache, int cache_cap, int batch,
                                int start_pos, const int32_t* positions, const void* next_attention_norm,
                                int input_normalised, void* ws, size_t ws_bytes, llama3_stream_t stream) {
  if (positions && (reinterpret_cast<uintptr_t>(positions) & 3)) return LLAMA3_ERR_ALIGN;
  if (next_attention_norm && !aligned16(next_attention_norm)) return LLAMA3_ERR_ALIGN;
  Workspace L;
  L3_TRY(check_layer_args(cfg, w, rope, rope_len, x, k_cache, v_cache, cache_cap, batch, 1, start_pos, ws,
                          ws_bytes, &L));
  cudaStream_t st = (cudaStream_t)stream;
  // Only the tcgen05 decode path hands the normalised input from block to
  // block; every other path ignores both flags and normalises x itself.
  if (use_tc(cfg) && (positions || batch <= 256))
    return layer_tc_decode(cfg, w, rope, x, k_cache, v_cache, cache_cap, batch, start_pos, L, ws, st, positions,
                           next_attention_norm, input_normalised != 0);
  if (positions)
    return llama3_layer_decode_ragged(cfg, w, rope, rope_len, x, k_cache, v_cache, cache_cap, batch, positions,
                                      start_pos, ws, ws_bytes, stream);
  return llama3_layer_decode(cfg, w, rope, rope_len, x, k_cache, v_cache, cache_cap, batch, start_pos, ws, ws_bytes,
                             stream);
}

int llama3_decode_step(const llama3_config* cfg, const llama3_layer_weights* layers, int n_layers,
                       const float* rope, int rope_len, void* x, void* const* k_caches, void* const* v_caches,
                       int cache_cap, int batch, int start_pos, const int32_t* positions, void* ws,
                       size_t ws_bytes, llama3_stream_t stream) {
  if (!layers || n_layers < 1 || !k_caches || !v_caches) return LLAMA3_ERR_ARG;
  if (positions && (reinterpret_cast<uintptr_t>(positions) & 3)) return LLAMA3_ERR_ALIGN;
  Workspace L;
  for (int i = 0; i < n_layers; ++i)
    L3_TRY(check_layer_args(cfg, &layers[i], rope, rope_len, x, k_caches[i], v_caches[i], cache_cap, batch, 1,
                            start_pos, ws, ws_bytes, &L));
  (void)L;
  // the block loop, each block handing the next one its normalised input
  for (int i = 0; i < n_layers; ++i) {
    const void* next_norm = i + 1 < n_layers ? layers[i + 1].attention_norm : nullptr;
    L3_TRY(llama3_layer_decode_chained(cfg, &layers[i], rope, rope_len, x, k_caches[i], v_caches[i], cache_cap,
                                       batch, start_pos, positions, next_norm, i > 0, ws, ws_bytes, stream));
  }
  return LLAMA3_OK;
}

int llama3_layer_forward_docs(const llama3_config* cfg, const llama3_layer_weights* w, const float* rope,
                              int rope_len, void* x, void* k_cache, void* v_cache, int cache_cap, int batch, int seq,
                              int start_pos, const int32_t* doc_start, void* ws, size_t ws_bytes,
                              llama3_stream_t stream) {
  Workspace L;
  L3_TRY(check_layer_args(cfg, w, rope, rope_len, x, k_cache, v_cache, cache_cap, batch, seq, start_pos, ws,
                          ws_bytes, &L));
  if (!doc_start) return LLAMA3_ERR_ARG;
  if (!aligned16(doc_start)) return LLAMA3_ERR_ALIGN;
  cudaStream_t st = (cudaStream_t)stream;
  if (use_tc(cfg))
    return layer_tc_prefill(cfg, w, rope, x, k_cache, v_cache, cache_cap, batch, seq, start_pos, L, ws, st,
                            doc_start);
  if (cfg->dtype == LLAMA3_DTYPE_F32)
    return layer_simt<float>(cfg, w, rope, x, k_cache, v_cache, cache_cap, batch, seq, start_pos, L, ws, st,
                             doc_start);
  return layer_simt<bf16>(cfg, w, rope, x, k_cache, v_cache, cache_cap, batch, seq, start_pos, L, ws, st,
                          doc_start);
}

int llama3_attention_docs(const llama3_config* cfg, const void* q, const void* k_cache, const void* v_cache,
                          int cache_cap, int batch, int seq, int start_pos, const int32_t* doc_start, void* out,
                          void* ws, size_t ws_bytes, llama3_stream_t stream) {
  L3_TRY(check_config(cfg));
  if (!q || !k_cache || !v_cache || !out || !doc_start || batch < 1 || seq < 1 || start_pos < 0)
    return LLAMA3_ERR_ARG;
  if ((long long)start_pos + seq > cache_cap) return LLAMA3_ERR_ARG;
  if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) || !aligned16(doc_start))
    return LLAMA3_ERR_ALIGN;
  Workspace L = layout(cfg, batch, seq, 1);
  if (!ws || ws_bytes < L.total) return LLAMA3_ERR_WORKSPACE;
  return attention_dispatch(cfg, q, k_cache, v_cache, cache_cap, batch, seq, start_pos, out,
                            ws_at<float>(ws, L.attn_part), (cudaStream_t)stream, doc_start);
}

int llama3_lm_head_argmax(const llama3_config* cfg, const void* norm_w, const void* w_out, const void* h, int rows,
                          long long row_stride, int32_t* ids_out, float* logits_out, void* ws, size_t ws_bytes,
                          llama3_stream_t stream) {
  L3_TRY(check_lm_head_args(cfg, norm_w, w_out, h, rows, row_stride, ids_out, logits_out));
  Workspace L = layout(cfg, 1, 1, rows);
  if (!ws || ws_bytes < L.total) return LLAMA3_ERR_WORKSPACE;
  if (!aligned16(ws)) return LLAMA3_ERR_ALIGN;
  return lm_head_run(cfg, norm_w, w_out, h, rows, row_stride, ids_out, logits_out, ws_at<void>(ws, L.lm_rows),
                     ws_at<unsigned long long>(ws, L.keys), (cudaStream_t)stream);
}

}  // extern "C"

// ===========================================================================
// LM head without a caller workspace: scratch in a fixed device global.
// ===========================================================================
// For callers that cannot hand the library device memory, this 4 MiB array
// takes the place of the workspace.  It exists on every device that loads the
// library.  Host code must not use the symbol as a pointer: its device
// address belongs to the current context and is looked up with
// cudaGetSymbolAddress.
static __device__ __align__(256) unsigned char g_noalloc_scratch[LLAMA3_NOALLOC_SCRATCH_BYTES];

namespace {
typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
struct NoallocSlot {
  CUcontext ctx;   // context the address was looked up in
  void* addr;
};
NoallocSlot g_noalloc[kMaxDevices];
std::mutex g_noalloc_mu;

int current_context(CUcontext* ctx) {
  static CtxGetCurrentFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return (CtxGetCurrentFn) nullptr;
    return reinterpret_cast<CtxGetCurrentFn>(p);
  }();
  if (!fn) return LLAMA3_ERR_CUDA;
  CUresult r = fn(ctx);
  if (r != CUDA_SUCCESS) {
    t_last_cuda = (int)r;
    return LLAMA3_ERR_CUDA;
  }
  return LLAMA3_OK;
}

// Device address of g_noalloc_scratch in the current context.  Outside a
// stream capture it is looked up on every call, so a context that was torn
// down and created again (cudaDeviceReset) gets its own address.  Inside a
// capture the address cached by an earlier call in the same context is used;
// without one the call fails instead of looking it up mid-capture.
int noalloc_scratch(cudaStream_t st, void** out) {
  int dev = 0;
  L3_TRY(current_device(&dev));
  cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
  L3_CUDA(cudaStreamIsCapturing(st, &cs));
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  NoallocSlot& slot = g_noalloc[dev];
  if (cs != cudaStreamCaptureStatusNone) {
    CUcontext ctx = nullptr;
    L3_TRY(current_context(&ctx));
    if (!slot.addr || slot.ctx != ctx) return LLAMA3_ERR_ARG;
    *out = slot.addr;
    return LLAMA3_OK;
  }
  // the lookup also makes the device's primary context current
  void* p = nullptr;
  L3_CUDA(cudaGetSymbolAddress(&p, g_noalloc_scratch));
  CUcontext ctx = nullptr;
  L3_TRY(current_context(&ctx));
  slot.ctx = ctx;
  slot.addr = p;
  *out = p;
  return LLAMA3_OK;
}
}  // namespace

extern "C" int llama3_lm_head_argmax_noalloc(const llama3_config* cfg, const void* norm_w, const void* w_out,
                                             const void* h, int rows, long long row_stride, int32_t* ids_out,
                                             float* logits_out, llama3_stream_t stream) {
  L3_TRY(check_lm_head_args(cfg, norm_w, w_out, h, rows, row_stride, ids_out, logits_out));
  const size_t keys_bytes = up256((size_t)rows * 8);
  const size_t rows_bytes = (size_t)rows * cfg->dim * esize(cfg);
  if (keys_bytes + rows_bytes > (size_t)LLAMA3_NOALLOC_SCRATCH_BYTES) return LLAMA3_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  void* base = nullptr;
  L3_TRY(noalloc_scratch(st, &base));
  // keys first (the previous call's maxima are overwritten by lm_head_run's
  // initialisation), then the normalised rows, 256-byte aligned
  unsigned long long* keys = reinterpret_cast<unsigned long long*>(base);
  void* hn = static_cast<char*>(base) + keys_bytes;
  return lm_head_run(cfg, norm_w, w_out, h, rows, row_stride, ids_out, logits_out, hn, keys, st);
}
