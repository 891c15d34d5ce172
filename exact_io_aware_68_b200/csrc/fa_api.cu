// The C ABI declared in include/fa.h: argument validation, TMA descriptor encoding and the
// kernel launches.  The kernels live in the headers included below; this is the library's
// single translation unit.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "../../include/fa.h"
#include "bwd_dq_sm100.cuh"
#include "bwd_sm100.cuh"
#include "decode_sm100.cuh"
#include "fwd256_sm100.cuh"
#include "fwd_sm100.cuh"
#include "simt_f32.cuh"

namespace {

thread_local char g_err[512] = "";

fa_status fail(fa_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

uint64_t default_wait_ns() {
  const char* e = std::getenv("FA_WAIT_LIMIT_MS");
  if (e != nullptr) {
    const long long ms = std::atoll(e);
    if (ms > 0) return uint64_t(ms) * 1000000ull;
  }
  return 2000000000ull;
}
std::atomic<uint64_t> g_wait_ns{default_wait_ns()};
std::atomic<int> g_debug_flags{0};

// cuTensorMapEncodeTiled from the driver, fetched through the runtime (no -lcuda needed).
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 3-D view {d, N, B*H} of a bf16 [B,H,N,d] tensor, loaded as 64 x box_rows x 1 boxes with the
// 128-byte swizzle; rows past N (the ragged last tile) read as zeros.
fa_status make_tile_map(CUtensorMap* map, const void* ptr, int BH, int N, int d, const char* name,
                        unsigned box_rows = 128) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(N), cuuint64_t(BH)};
  const cuuint64_t strides[2] = {cuuint64_t(d) * 2, cuuint64_t(N) * cuuint64_t(d) * 2};
  const cuuint32_t box[3] = {64, box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled(%s) failed with CUresult %d", name, int(r));
  return FA_OK;
}

// 3-D view {d, N, B*H} of the fp32 dQ accumulator for the backward's TMA bulk reductions:
// boxes of (features per dQ warp) x (queries per round), no swizzle; rows past N are not written.
fa_status make_dq_map(CUtensorMap* map, const void* ptr, int BH, int N, int d, unsigned box_x, unsigned box_y) {
  auto fn = encode_fn();
  if (fn == nullptr) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled is unavailable from the driver");
  const cuuint64_t dims[3] = {cuuint64_t(d), cuuint64_t(N), cuuint64_t(BH)};
  const cuuint64_t strides[2] = {cuuint64_t(d) * 4, cuuint64_t(N) * cuuint64_t(d) * 4};
  const cuuint32_t box[3] = {box_x, box_y, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<void*>(ptr), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(FA_ERR_CUDA, "cuTensorMapEncodeTiled(dQ accumulator) failed with CUresult %d", int(r));
  return FA_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Which head dimensions an entry point takes.
enum class Dims { kBf16, kBf16Fwd, kF32 };

fa_status check_common(int B, int H, int N, int d, float scale, float dropout_p, Dims dims) {
  if (B < 1 || H < 1 || N < 1) return fail(FA_ERR_INVALID_ARG, "B, H and N must be >= 1 (got %d, %d, %d)", B, H, N);
  if (int64_t(B) * H > 65535) return fail(FA_ERR_UNSUPPORTED, "B*H = %lld exceeds 65535", (long long)B * H);
  if (int64_t(N) > (int64_t(1) << 30)) return fail(FA_ERR_UNSUPPORTED, "N = %d is too large", N);
  if (dims == Dims::kBf16 && d != 64 && d != 128)
    return fail(FA_ERR_UNSUPPORTED, "head dimension d = %d: this bf16 entry point supports d in {64, 128}", d);
  if (dims == Dims::kBf16Fwd && d != 64 && d != 128 && d != 256)
    return fail(FA_ERR_UNSUPPORTED, "head dimension d = %d: the bf16 forward supports d in {64, 128, 256}", d);
  if (dims == Dims::kF32 && (d < 1 || d > 128))
    return fail(FA_ERR_UNSUPPORTED, "head dimension d = %d: fp32 supports 1 <= d <= 128", d);
  if (!std::isfinite(scale) || !(scale > 0.f)) return fail(FA_ERR_INVALID_ARG, "scale must be finite and > 0");
  if (!(dropout_p >= 0.f) || !(dropout_p < 1.f)) return fail(FA_ERR_INVALID_ARG, "dropout_p must be in [0, 1)");
  return FA_OK;
}

#define FA_CHECK_PTR(p)                                                                      \
  do {                                                                                       \
    if ((p) == nullptr) return fail(FA_ERR_INVALID_ARG, "%s is NULL", #p);                   \
    if (!aligned16(p)) return fail(FA_ERR_INVALID_ARG, "%s is not 16-byte aligned", #p);     \
  } while (0)

fa_status launch_status(const char* what) {
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
  return FA_OK;
}

// The 15-bit dropout threshold: a column is kept when its 15-bit draw is >= this value.
uint32_t drop_threshold(float p) {
  const double t = std::floor(double(p) * 32768.0);
  return uint32_t(t > 32767.0 ? 32767.0 : t);
}

struct Workspace {
  float* dq_acc;
  float* dvec;
  unsigned int* work_ctr;
};
size_t ws_dq_bytes(int B, int H, int N, int d) {
  return (size_t(B) * H * N * d * 4 + 255) & ~size_t(255);
}
size_t ws_d_bytes(int B, int H, int N) { return (size_t(B) * H * N * 4 + 255) & ~size_t(255); }
// fp32 dQ accumulator, D, and 256 bytes for the main kernel's item counter
size_t ws_total_bytes(int B, int H, int N, int d) { return ws_dq_bytes(B, H, N, d) + ws_d_bytes(B, H, N) + 256; }
fa_status check_workspace(void* ws, size_t bytes, int B, int H, int N, int d, Workspace* out) {
  if (ws == nullptr) return fail(FA_ERR_INVALID_ARG, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return fail(FA_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  const size_t need = ws_total_bytes(B, H, N, d);
  if (bytes < need) return fail(FA_ERR_INVALID_ARG, "workspace has %zu bytes, needs %zu", bytes, need);
  out->dq_acc = static_cast<float*>(ws);
  out->dvec = reinterpret_cast<float*>(static_cast<char*>(ws) + ws_dq_bytes(B, H, N, d));
  out->work_ctr =
      reinterpret_cast<unsigned int*>(static_cast<char*>(ws) + ws_dq_bytes(B, H, N, d) + ws_d_bytes(B, H, N));
  return FA_OK;
}

// Number of SMs of the current device (queried once per device).
fa_status sm_count(int* out) {
  static std::atomic<int> cache[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev >= 0 && dev < 64 && cache[dev].load() > 0) {
    *out = cache[dev].load();
    return FA_OK;
  }
  int n = 0;
  e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess || n <= 0) return fail(FA_ERR_CUDA, "cudaDeviceGetAttribute(SM count): %s", cudaGetErrorString(e));
  if (dev >= 0 && dev < 64) cache[dev].store(n);
  *out = n;
  return FA_OK;
}

// L2 size of the current device in bytes (queried once per device).
fa_status l2_bytes(size_t* out) {
  static std::atomic<long long> cache[64];
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev >= 0 && dev < 64 && cache[dev].load() > 0) {
    *out = size_t(cache[dev].load());
    return FA_OK;
  }
  int n = 0;
  e = cudaDeviceGetAttribute(&n, cudaDevAttrL2CacheSize, dev);
  if (e != cudaSuccess || n <= 0) return fail(FA_ERR_CUDA, "cudaDeviceGetAttribute(L2 size): %s", cudaGetErrorString(e));
  if (dev >= 0 && dev < 64) cache[dev].store(n);
  *out = size_t(n);
  return FA_OK;
}

template <typename K>
fa_status set_smem(K kernel, int bytes) {
  const cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "cudaFuncSetAttribute: %s", cudaGetErrorString(e));
  return FA_OK;
}

// The warp-specialised kernels re-split their registers per warpgroup with setmaxnreg; the split
// adds up to `regs` registers per thread at launch.  A build whose kernel was given fewer
// registers would leave a setmaxnreg.inc waiting forever, so it is refused before the launch.
template <typename K>
fa_status check_launch_regs(K kernel, int regs, const char* name) {
  cudaFuncAttributes a{};
  const cudaError_t e = cudaFuncGetAttributes(&a, kernel);
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "cudaFuncGetAttributes(%s): %s", name, cudaGetErrorString(e));
  if (a.numRegs < regs)
    return fail(FA_ERR_INTERNAL, "%s was built with %d registers per thread; its register split needs %d", name,
                a.numRegs, regs);
  return FA_OK;
}

template <int D, bool DROPOUT>
fa_status launch_fwd(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const fa::FwdParams& p,
                     cudaStream_t s) {
  using L = fa::FwdLayout<D>;
  fa_status st = set_smem(fa::fa_fwd_sm100_kernel<D, DROPOUT>, L::BYTES);
  if (st != FA_OK) return st;
  if ((st = check_launch_regs(fa::fa_fwd_sm100_kernel<D, DROPOUT>, fa::kFwdLaunchRegs, "fa_fwd kernel")) != FA_OK)
    return st;
  // persistent: one CTA per SM (or fewer when there are fewer work items)
  const long long items = (long long)p.n_pairs * p.B * p.H;
  int sms = 0;
  if ((st = sm_count(&sms)) != FA_OK) return st;
  const dim3 grid(unsigned(items < sms ? items : sms));
  fa::fa_fwd_sm100_kernel<D, DROPOUT><<<grid, fa::kFwdThreads, L::BYTES, s>>>(mq, mk, mv, p);
  return launch_status("fa_fwd kernel launch");
}

template <int D, bool DROPOUT, bool DQ>
fa_status launch_bwd_main(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                          fa::BwdParams p, cudaStream_t s) {
  using L = fa::BwdLayout<D, DROPOUT>;
  CUtensorMap mdq;
  fa_status st0 = make_dq_map(&mdq, p.dq_acc, p.B * p.H, p.N, D, L::FPW, L::QPR);
  if (st0 != FA_OK) return st0;
  fa_status st = set_smem(fa::fa_bwd_sm100_kernel<D, DROPOUT, DQ>, L::BYTES);
  if (st != FA_OK) return st;
  if ((st = check_launch_regs(fa::fa_bwd_sm100_kernel<D, DROPOUT, DQ>, fa::kBwdLaunchRegs, "fa_bwd main kernel")) !=
      FA_OK)
    return st;
  int sms = 0;
  if ((st = sm_count(&sms)) != FA_OK) return st;
  // Items (head, key tile) are taken in a linear launch order. Head-major order keeps the CTAs
  // in flight on a few heads, so their Q and dO stay in L2, but each head's heaviest causal key
  // tile starts only when the head does. That tail is about 2 * SMs / (B*H*n_tiles) of the run.
  // While there are at most 20 items per SM, the order is instead: groups of heads one after
  // another, key-tile-major inside each group. Every head's first key tile (the most query
  // tiles when causal) then starts with its group, and the one-tile items form each group's tail.
  // A group holds at most 16 heads, and its Q, dO and fp32 dQ accumulator (8*N*d bytes a head)
  // fit in 32 MB of L2. Measured on the headline causal 2x16x4096x128: head-major 352 us,
  // key-tile-major over all 32 heads 332-340 us (2.6x the algorithmic DRAM bytes), groups of 8
  // heads 330 us. 64k-token sequences keep head-major (the other order was 9 % slower). The group
  // size comes from the device's L2 size (fa_bwd_head_group).
  p.kt_major = int64_t(p.B) * p.H * p.n_tiles <= 20 * int64_t(sms) ? 1 : 0;
  size_t l2 = 0;
  if ((st = l2_bytes(&l2)) != FA_OK) return st;
  p.head_group = fa_bwd_head_group(p.N, D, l2);
  // persistent: one CTA per SM (or fewer when there are fewer items), each walking items
  // c, c + G, c + 2G, ... of the launch order
  const long long items = (long long)p.B * p.H * p.n_tiles;
  const dim3 grid(unsigned(items < sms ? items : sms));
  fa::fa_bwd_sm100_kernel<D, DROPOUT, DQ><<<grid, fa::kBwdThreads, L::BYTES, s>>>(mq, mk, mv, mdo, mdq, p);
  return launch_status("fa_bwd main kernel launch");
}

template <int D, bool DROPOUT>
fa_status launch_dq_pass(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const CUtensorMap& mdo,
                         const fa::DqParams& p, dim3 grid, cudaStream_t s) {
  using L = fa::DqLayout<D>;
  const fa_status st = set_smem(fa::fa_bwd_dq_pass_kernel<D, DROPOUT>, L::BYTES);
  if (st != FA_OK) return st;
  fa::fa_bwd_dq_pass_kernel<D, DROPOUT><<<grid, 256, L::BYTES, s>>>(mq, mk, mv, mdo, p);
  return launch_status("fa_bwd_split dQ kernel launch");
}

fa::BwdParams bwd_params(int B, int H, int N, float scale, int causal, const int32_t* key_lens, float dropout_p,
                         uint64_t seed, const Workspace& w) {
  fa::BwdParams p{};
  p.lse = nullptr;
  p.dvec = w.dvec;
  p.dq_acc = w.dq_acc;
  p.work_ctr = w.work_ctr;
  p.key_lens = key_lens;
  p.B = B;
  p.H = H;
  p.N = N;
  p.n_tiles = (N + 127) / 128;
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.dropout = dropout_p > 0.f ? 1 : 0;
  p.drop_thr = drop_threshold(dropout_p);
  p.drop_scale = dropout_p > 0.f ? 1.f / (1.f - dropout_p) : 1.f;
  p.seed = seed;
  p.wait_ns = g_wait_ns.load();
  p.debug_flags = g_debug_flags.load();
  return p;
}

// Key-range split of the decode kernel.  Its shared memory holds one CTA per SM, so a grid of
// BH * n CTAs runs in ceil(BH * n / sms) waves, each as long as one split's keys.  n minimises
// waves * (chunk + 256): the 256 stands for a split's fixed cost (Q load, pipeline fill, partial
// write) in keys.  Chunks are whole 128-key blocks of at least 512 keys; n <= 4 * sms.  With no SM
// count (sms <= 0) the split is the finest one, n = ceil(Nkv / 512), which bounds the workspace of
// every device.  Host arithmetic only.
struct DecodeSplit {
  int chunk, n_split;
};
DecodeSplit decode_split(int BH, int Nkv, int sms) {
  auto chunk_for = [&](long long n) {
    long long c = (Nkv + n - 1) / n;
    c = (c + 127) / 128 * 128;
    return c < 512 ? 512LL : c;
  };
  const long long finest = (Nkv + 511) / 512;
  if (sms <= 0) {
    const long long c = chunk_for(finest);
    return DecodeSplit{int(c), int((Nkv + c - 1) / c)};
  }
  const long long top = std::min<long long>(finest, 4LL * sms);
  DecodeSplit best{0, 0};
  long long best_cost = -1;
  for (long long n = 1; n <= top; ++n) {
    const long long c = chunk_for(n);
    const long long splits = (Nkv + c - 1) / c;
    const long long waves = (BH * splits + sms - 1) / sms;
    const long long cost = waves * (c + 256);
    if (best_cost < 0 || cost < best_cost) {
      best_cost = cost;
      best = DecodeSplit{int(c), int(splits)};
    }
  }
  return best;
}
// SM count of the current device for the decode split, or 0 with no visible device (the CUDA error
// that the query leaves is cleared, and the library's error message is left alone).
int decode_sms() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}
size_t decode_o_bytes(int BH, int n_split, int Nq, int d) {
  return (size_t(BH) * n_split * Nq * d * 4 + 255) & ~size_t(255);
}
// Two partials per split (one per key half of the split kernel's tile).
size_t decode_ws_bytes(int BH, int Nq, int Nkv, int d, int sms) {
  const DecodeSplit sp = decode_split(BH, Nkv, sms);
  const int n_part = 2 * sp.n_split;
  return decode_o_bytes(BH, n_part, Nq, d) + ((size_t(BH) * n_part * Nq * 2 * 4 + 255) & ~size_t(255));
}

template <int D>
fa_status launch_decode(const CUtensorMap& mq, const CUtensorMap& mk, const CUtensorMap& mv, const fa::DecodeParams& p,
                        cudaStream_t s) {
  using L = fa::DecodeLayout<D>;
  fa_status st = set_smem(fa::fa_decode_split_kernel<D>, L::BYTES);
  if (st != FA_OK) return st;
  fa::fa_decode_split_kernel<D><<<dim3(p.n_split, p.B * p.H), 192, L::BYTES, s>>>(mq, mk, mv, p);
  if ((st = launch_status("fa_fwd_decode split kernel launch")) != FA_OK) return st;
  // The combine is a programmatic dependent launch: it may be scheduled while the split kernel
  // runs and waits (griddepcontrol.wait) until that grid has completed and its writes are visible,
  // so the second launch adds no gap of its own.
  const unsigned rows = unsigned(p.B * p.H * p.Nq);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((rows + 7) / 8);
  cfg.blockDim = dim3(256);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, fa::fa_decode_combine_kernel<D>, p);
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "fa_fwd_decode combine kernel launch: %s", cudaGetErrorString(e));
  return launch_status("fa_fwd_decode combine kernel launch");
}

// The d = 256 forward (fwd256_sm100.cuh): one query tile per CTA, 64-key blocks, persistent grid.
fa_status fwd256(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, float scale,
                 int causal, const int32_t* key_lens, float dropout_p, uint64_t seed, cudaStream_t s) {
  using L = fa::Fwd256Layout;
  CUtensorMap mq, mk, mv;
  fa_status st;
  if ((st = make_tile_map(&mq, q, B * H, N, 256, "q")) != FA_OK) return st;
  if ((st = make_tile_map(&mk, k, B * H, N, 256, "k", 64)) != FA_OK) return st;
  if ((st = make_tile_map(&mv, v, B * H, N, 256, "v", 64)) != FA_OK) return st;
  fa::Fwd256Params p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.key_lens = key_lens;
  p.B = B;
  p.H = H;
  p.N = N;
  p.n_qtiles = (N + 127) / 128;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.dropout = dropout_p > 0.f ? 1 : 0;
  p.drop_thr = drop_threshold(dropout_p);
  p.drop_scale = dropout_p > 0.f ? 1.f / (1.f - dropout_p) : 1.f;
  p.seed = seed;
  p.wait_ns = g_wait_ns.load();
  int sms = 0;
  if ((st = sm_count(&sms)) != FA_OK) return st;
  const long long items = (long long)p.n_qtiles * B * H;
  const dim3 grid(unsigned(items < sms ? items : sms));
  if (p.dropout) {
    if ((st = set_smem(fa::fa_fwd256_sm100_kernel<true>, L::BYTES)) != FA_OK) return st;
    fa::fa_fwd256_sm100_kernel<true><<<grid, 256, L::BYTES, s>>>(mq, mk, mv, p);
  } else {
    if ((st = set_smem(fa::fa_fwd256_sm100_kernel<false>, L::BYTES)) != FA_OK) return st;
    fa::fa_fwd256_sm100_kernel<false><<<grid, 256, L::BYTES, s>>>(mq, mk, mv, p);
  }
  return launch_status("fa_fwd (d = 256) kernel launch");
}

unsigned grid_for(uint64_t work, unsigned per_block) {
  const uint64_t g = (work + per_block - 1) / per_block;
  return unsigned(g < 1 ? 1 : (g > (1u << 30) ? (1u << 30) : g));
}

}  // namespace

extern "C" {

int fa_bwd_head_group(int N, int d, size_t l2_bytes) {
  // Q, dO (bf16) and the fp32 dQ accumulator of one head: 8 * N * d bytes.  A group fills about a
  // quarter of L2, rounded to the nearest whole head (measured best on the 126 MB B200: groups of 8
  // heads at N = 4096, d = 128), 1..16 heads.
  if (N < 1 || d < 1) return 1;
  const uint64_t per_head = 8ull * uint64_t(N) * uint64_t(d);
  const uint64_t g = (uint64_t(l2_bytes) / 4 + per_head / 2) / per_head;
  return int(g < 1 ? 1 : (g > 16 ? 16 : g));
}

fa_status fa_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int N, int d,
                 float scale, int causal, const int32_t* key_lens, float dropout_p, uint64_t seed, cudaStream_t stream) {
  fa_status st = check_common(B, H, N, d, scale, dropout_p, Dims::kBf16Fwd);
  if (st != FA_OK) return st;
  FA_CHECK_PTR(q);
  FA_CHECK_PTR(k);
  FA_CHECK_PTR(v);
  FA_CHECK_PTR(o);
  FA_CHECK_PTR(lse);
  if (d == 256) return fwd256(q, k, v, o, lse, B, H, N, scale, causal, key_lens, dropout_p, seed, stream);
  CUtensorMap mq, mk, mv;
  if ((st = make_tile_map(&mq, q, B * H, N, d, "q")) != FA_OK) return st;
  if ((st = make_tile_map(&mk, k, B * H, N, d, "k")) != FA_OK) return st;
  if ((st = make_tile_map(&mv, v, B * H, N, d, "v")) != FA_OK) return st;
  fa::FwdParams p{};
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.key_lens = key_lens;
  p.B = B;
  p.H = H;
  p.N = N;
  p.n_qtiles = (N + 127) / 128;
  p.n_pairs = (p.n_qtiles + 1) / 2;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.dropout = dropout_p > 0.f ? 1 : 0;
  p.drop_thr = drop_threshold(dropout_p);
  p.drop_scale = dropout_p > 0.f ? 1.f / (1.f - dropout_p) : 1.f;
  p.seed = seed;
  p.wait_ns = g_wait_ns.load();
  p.debug_flags = g_debug_flags.load();
  p.o_align32 = (reinterpret_cast<uintptr_t>(o) & 31u) == 0 ? 1 : 0;
  cudaStream_t s = stream;
  if (d == 64) return p.dropout ? launch_fwd<64, true>(mq, mk, mv, p, s) : launch_fwd<64, false>(mq, mk, mv, p, s);
  return p.dropout ? launch_fwd<128, true>(mq, mk, mv, p, s) : launch_fwd<128, false>(mq, mk, mv, p, s);
}

fa_status fa_fwd_f32(const float* q, const float* k, const float* v, float* o, float* lse, int B, int H, int N, int d,
                     float scale, int causal, const int32_t* key_lens, float dropout_p, uint64_t seed, cudaStream_t stream) {
  fa_status st = check_common(B, H, N, d, scale, dropout_p, Dims::kF32);
  if (st != FA_OK) return st;
  FA_CHECK_PTR(q);
  FA_CHECK_PTR(k);
  FA_CHECK_PTR(v);
  FA_CHECK_PTR(o);
  FA_CHECK_PTR(lse);
  fa::F32Params p{};
  p.q = q;
  p.k = k;
  p.v = v;
  p.o = o;
  p.lse = lse;
  p.key_lens = key_lens;
  p.B = B;
  p.H = H;
  p.N = N;
  p.d = d;
  p.causal = causal ? 1 : 0;
  p.scale = scale;
  p.dropout = dropout_p > 0.f ? 1 : 0;
  p.drop_thr = drop_threshold(dropout_p);
  p.drop_scale = dropout_p > 0.f ? 1.f / (1.f - dropout_p) : 1.f;
  p.seed = seed;
  cudaStream_t s = stream;
  const dim3 grid((N + 63) / 64, B * H);   // 64 query rows per CTA
  if (d <= 32)
    fa::fa_fwd_f32_kernel<32><<<grid, 128, 0, s>>>(p);
  else if (d <= 64)
    fa::fa_fwd_f32_kernel<64><<<grid, 128, 0, s>>>(p);
  else if (d <= 96)
    fa::fa_fwd_f32_kernel<96><<<grid, 128, 0, s>>>(p);
  else
    fa::fa_fwd_f32_kernel<128><<<grid, 128, 0, s>>>(p);
  return launch_status("fa_fwd_f32 kernel launch");
}

size_t fa_bwd_workspace_size(int B, int H, int N, int d) {
  if (B < 1 || H < 1 || N < 1 || d < 1) return 0;
  return ws_total_bytes(B, H, N, d);
}

fa_status fa_bwd_prep(const void* o, const void* dO, int B, int H, int N, int d, void* workspace,
                      size_t workspace_bytes, cudaStream_t stream) {
  fa_status st = check_common(B, H, N, d, 1.f, 0.f, Dims::kBf16);
  if (st != FA_OK) return st;
  FA_CHECK_PTR(o);
  FA_CHECK_PTR(dO);
  Workspace w;
  if ((st = check_workspace(workspace, workspace_bytes, B, H, N, d, &w)) != FA_OK) return st;
  fa::BwdParams p = bwd_params(B, H, N, 1.f, 0, nullptr, 0.f, 0, w);
  p.o = static_cast<const __nv_bfloat16*>(o);
  p.dO = static_cast<const __nv_bfloat16*>(dO);
  cudaStream_t s = stream;
  const uint64_t threads = uint64_t(B) * H * N * (d / 8);
  if (d == 64)
    fa::fa_bwd_prep_kernel<64><<<grid_for(threads, 256), 256, 0, s>>>(p);
  else
    fa::fa_bwd_prep_kernel<128><<<grid_for(threads, 256), 256, 0, s>>>(p);
  return launch_status("fa_bwd_prep kernel launch");
}

fa_status fa_bwd_main(const void* q, const void* k, const void* v, const float* lse, const void* dO, void* dk, void* dv,
                      int B, int H, int N, int d, float scale, int causal, const int32_t* key_lens, float dropout_p,
                      uint64_t seed, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  fa_status st = check_common(B, H, N, d, scale, dropout_p, Dims::kBf16);
  if (st != FA_OK) return st;
  FA_CHECK_PTR(q);
  FA_CHECK_PTR(k);
  FA_CHECK_PTR(v);
  FA_CHECK_PTR(lse);
  FA_CHECK_PTR(dO);
  FA_CHECK_PTR(dk);
  FA_CHECK_PTR(dv);
  Workspace w;
  if ((st = check_workspace(workspace, workspace_bytes, B, H, N, d, &w)) != FA_OK) return st;
  CUtensorMap mq, mk, mv, mdo;
  if ((st = make_tile_map(&mq, q, B * H, N, d, "q")) != FA_OK) return st;
  if ((st = make_tile_map(&mk, k, B * H, N, d, "k")) != FA_OK) return st;
  if ((st = make_tile_map(&mv, v, B * H, N, d, "v")) != FA_OK) return st;
  if ((st = make_tile_map(&mdo, dO, B * H, N, d, "dO")) != FA_OK) return st;
  fa::BwdParams p = bwd_params(B, H, N, scale, causal, key_lens, dropout_p, seed, w);
  p.lse = lse;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.out_align32 = ((reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv)) & 31u) == 0 ? 1 : 0;
  cudaStream_t s = stream;
  if (d == 64)
    return p.dropout ? launch_bwd_main<64, true, true>(mq, mk, mv, mdo, p, s)
                     : launch_bwd_main<64, false, true>(mq, mk, mv, mdo, p, s);
  return p.dropout ? launch_bwd_main<128, true, true>(mq, mk, mv, mdo, p, s)
                   : launch_bwd_main<128, false, true>(mq, mk, mv, mdo, p, s);
}

fa_status fa_bwd_split(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                       void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                       const int32_t* key_lens, float dropout_p, uint64_t seed, void* workspace, size_t workspace_bytes,
                       cudaStream_t stream) {
  fa_status st = check_common(B, H, N, d, scale, dropout_p, Dims::kBf16);
  if (st != FA_OK) return st;
  FA_CHECK_PTR(q);
  FA_CHECK_PTR(k);
  FA_CHECK_PTR(v);
  FA_CHECK_PTR(lse);
  FA_CHECK_PTR(dO);
  FA_CHECK_PTR(dq);
  FA_CHECK_PTR(dk);
  FA_CHECK_PTR(dv);
  Workspace w;
  if ((st = check_workspace(workspace, workspace_bytes, B, H, N, d, &w)) != FA_OK) return st;
  if ((st = fa_bwd_prep(o, dO, B, H, N, d, workspace, workspace_bytes, stream)) != FA_OK) return st;
  CUtensorMap mq, mk, mv, mdo;
  if ((st = make_tile_map(&mq, q, B * H, N, d, "q")) != FA_OK) return st;
  if ((st = make_tile_map(&mk, k, B * H, N, d, "k")) != FA_OK) return st;
  if ((st = make_tile_map(&mv, v, B * H, N, d, "v")) != FA_OK) return st;
  if ((st = make_tile_map(&mdo, dO, B * H, N, d, "dO")) != FA_OK) return st;
  // dK and dV: the main kernel without its dQ part
  fa::BwdParams p = bwd_params(B, H, N, scale, causal, key_lens, dropout_p, seed, w);
  p.lse = lse;
  p.dk = static_cast<__nv_bfloat16*>(dk);
  p.dv = static_cast<__nv_bfloat16*>(dv);
  p.out_align32 = ((reinterpret_cast<uintptr_t>(dk) | reinterpret_cast<uintptr_t>(dv)) & 31u) == 0 ? 1 : 0;
  if (d == 64)
    st = p.dropout ? launch_bwd_main<64, true, false>(mq, mk, mv, mdo, p, stream)
                   : launch_bwd_main<64, false, false>(mq, mk, mv, mdo, p, stream);
  else
    st = p.dropout ? launch_bwd_main<128, true, false>(mq, mk, mv, mdo, p, stream)
                   : launch_bwd_main<128, false, false>(mq, mk, mv, mdo, p, stream);
  if (st != FA_OK) return st;
  // dQ: its own pass, query-tile-major
  fa::DqParams dp{};
  dp.dq = static_cast<__nv_bfloat16*>(dq);
  dp.lse = lse;
  dp.dvec = w.dvec;
  dp.key_lens = key_lens;
  dp.B = B;
  dp.H = H;
  dp.N = N;
  dp.n_qtiles = (N + 127) / 128;
  dp.causal = causal ? 1 : 0;
  dp.scale = scale;
  dp.scale_log2 = scale * 1.4426950408889634f;
  dp.dropout = dropout_p > 0.f ? 1 : 0;
  dp.drop_thr = drop_threshold(dropout_p);
  dp.drop_scale = dropout_p > 0.f ? 1.f / (1.f - dropout_p) : 1.f;
  dp.seed = seed;
  dp.wait_ns = g_wait_ns.load();
  int sms = 0;
  if ((st = sm_count(&sms)) != FA_OK) return st;
  const long long items = (long long)dp.n_qtiles * B * H;
  const dim3 grid(unsigned(items < sms ? items : sms));
  if (d == 64)
    return dp.dropout ? launch_dq_pass<64, true>(mq, mk, mv, mdo, dp, grid, stream)
                      : launch_dq_pass<64, false>(mq, mk, mv, mdo, dp, grid, stream);
  return dp.dropout ? launch_dq_pass<128, true>(mq, mk, mv, mdo, dp, grid, stream)
                    : launch_dq_pass<128, false>(mq, mk, mv, mdo, dp, grid, stream);
}

fa_status fa_bwd_dq_convert(void* dq, int B, int H, int N, int d, float scale, void* workspace,
                            size_t workspace_bytes, cudaStream_t stream) {
  fa_status st = check_common(B, H, N, d, scale, 0.f, Dims::kBf16);
  if (st != FA_OK) return st;
  FA_CHECK_PTR(dq);
  Workspace w;
  if ((st = check_workspace(workspace, workspace_bytes, B, H, N, d, &w)) != FA_OK) return st;
  fa::BwdParams p = bwd_params(B, H, N, scale, 0, nullptr, 0.f, 0, w);
  p.dq = static_cast<__nv_bfloat16*>(dq);
  cudaStream_t s = stream;
  const uint64_t n8 = uint64_t(B) * H * N * d / 8;
  int sms = 0;
  if ((st = sm_count(&sms)) != FA_OK) return st;
  const unsigned cap = unsigned(sms) * 16u;   // grid-stride loop: 16 blocks of 256 threads per SM
  const unsigned grid = grid_for(n8, 256) > cap ? cap : grid_for(n8, 256);
  if (d == 64)
    fa::fa_bwd_dq_kernel<64><<<grid, 256, 0, s>>>(p);
  else
    fa::fa_bwd_dq_kernel<128><<<grid, 256, 0, s>>>(p);
  return launch_status("fa_bwd_dq_convert kernel launch");
}

fa_status fa_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO, void* dq,
                 void* dk, void* dv, int B, int H, int N, int d, float scale, int causal, const int32_t* key_lens,
                 float dropout_p, uint64_t seed, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  FA_CHECK_PTR(dq);
  fa_status st = fa_bwd_prep(o, dO, B, H, N, d, workspace, workspace_bytes, stream);
  if (st != FA_OK) return st;
  st = fa_bwd_main(q, k, v, lse, dO, dk, dv, B, H, N, d, scale, causal, key_lens, dropout_p, seed, workspace,
                   workspace_bytes, stream);
  if (st != FA_OK) return st;
  return fa_bwd_dq_convert(dq, B, H, N, d, scale, workspace, workspace_bytes, stream);
}

size_t fa_fwd_decode_workspace_size(int B, int H, int Nq, int Nkv, int d) {
  if (B < 1 || H < 1 || Nq < 1 || Nkv < 1 || d < 1) return 0;
  return decode_ws_bytes(B * H, Nq, Nkv, d, decode_sms());
}

int fa_fwd_decode_split(int B, int H, int Nkv, int sms) {
  if (B < 1 || H < 1 || Nkv < 1) return 0;
  return decode_split(B * H, Nkv, sms).n_split;
}

fa_status fa_fwd_decode(const void* q, const void* k, const void* v, void* o, float* lse, int B, int H, int Nq,
                        int Nkv, int d, float scale, int causal, const int32_t* key_lens, void* workspace,
                        size_t workspace_bytes, cudaStream_t stream) {
  fa_status st = check_common(B, H, Nkv, d, scale, 0.f, Dims::kBf16);
  if (st != FA_OK) return st;
  if (Nq < 1 || Nq > 64) return fail(FA_ERR_UNSUPPORTED, "Nq = %d: fa_fwd_decode takes 1 <= Nq <= 64", Nq);
  FA_CHECK_PTR(q);
  FA_CHECK_PTR(k);
  FA_CHECK_PTR(v);
  FA_CHECK_PTR(o);
  FA_CHECK_PTR(lse);
  if (workspace == nullptr) return fail(FA_ERR_INVALID_ARG, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(FA_ERR_INVALID_ARG, "workspace is not 256-byte aligned");
  const int sms = decode_sms();
  const size_t need = decode_ws_bytes(B * H, Nq, Nkv, d, sms);
  if (workspace_bytes < need) return fail(FA_ERR_INVALID_ARG, "workspace has %zu bytes, needs %zu", workspace_bytes, need);
  const DecodeSplit sp = decode_split(B * H, Nkv, sms);
  CUtensorMap mq, mk, mv;
  if ((st = make_tile_map(&mq, q, B * H, Nq, d, "q", 64)) != FA_OK) return st;
  if ((st = make_tile_map(&mk, k, B * H, Nkv, d, "k")) != FA_OK) return st;
  if ((st = make_tile_map(&mv, v, B * H, Nkv, d, "v")) != FA_OK) return st;
  fa::DecodeParams p{};
  p.part_o = static_cast<float*>(workspace);
  p.part_ml = reinterpret_cast<float*>(static_cast<char*>(workspace) + decode_o_bytes(B * H, 2 * sp.n_split, Nq, d));
  p.o = static_cast<__nv_bfloat16*>(o);
  p.lse = lse;
  p.key_lens = key_lens;
  p.B = B;
  p.H = H;
  p.Nq = Nq;
  p.Nkv = Nkv;
  p.chunk = sp.chunk;
  p.n_split = sp.n_split;
  p.n_part = 2 * sp.n_split;
  p.causal = causal ? 1 : 0;
  p.scale_log2 = scale * 1.4426950408889634f;
  p.wait_ns = g_wait_ns.load();
  return d == 64 ? launch_decode<64>(mq, mk, mv, p, stream) : launch_decode<128>(mq, mk, mv, p, stream);
}

fa_status fa_dropout_mask(uint8_t* keep, int B, int H, int N, float dropout_p, uint64_t seed, cudaStream_t stream) {
  if (keep == nullptr) return fail(FA_ERR_INVALID_ARG, "keep is NULL");
  if (B < 1 || H < 1 || N < 1) return fail(FA_ERR_INVALID_ARG, "B, H and N must be >= 1");
  if (!(dropout_p >= 0.f) || !(dropout_p < 1.f)) return fail(FA_ERR_INVALID_ARG, "dropout_p must be in [0, 1)");
  const uint64_t total = uint64_t(B) * H * N * uint64_t(N);
  cudaStream_t s = stream;
  int sms = 0;
  const fa_status st = sm_count(&sms);
  if (st != FA_OK) return st;
  const unsigned cap = unsigned(sms) * 32u;   // grid-stride loop: 32 blocks of 256 threads per SM
  const unsigned grid = grid_for(total, 256) > cap ? cap : grid_for(total, 256);
  fa::fa_dropout_mask_kernel<<<grid, 256, 0, s>>>(keep, total, N, seed, drop_threshold(dropout_p));
  return launch_status("fa_dropout_mask kernel launch");
}

fa_status fa_test_exp2_fma(const float* x, float* y, int n, cudaStream_t stream) {
  if (x == nullptr || y == nullptr) return fail(FA_ERR_INVALID_ARG, "x or y is NULL");
  if (n < 1) return fail(FA_ERR_INVALID_ARG, "n must be >= 1");
  fa::fa_exp2_fma_test_kernel<<<grid_for((uint64_t(n) + 1) / 2, 256), 256, 0, stream>>>(x, y, n);
  return launch_status("fa_test_exp2_fma kernel launch");
}

fa_status fa_check(cudaStream_t stream) {
  cudaError_t e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "cudaStreamSynchronize: %s", cudaGetErrorString(e));
  int code = 0;
  e = cudaMemcpyFromSymbol(&code, fa::g_fa_device_status, sizeof(int));
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "reading the device status word: %s", cudaGetErrorString(e));
  if (code == 0) return FA_OK;
  const int zero = 0;
  e = cudaMemcpyToSymbol(fa::g_fa_device_status, &zero, sizeof(int));
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "clearing the device status word: %s", cudaGetErrorString(e));
  if (code == fa::kStatusTimeout) return fail(FA_ERR_TIMEOUT, "a kernel's bounded wait ran out");
  return fail(FA_ERR_INTERNAL, "device status %d (dynamic shared memory not 1024-byte aligned)", code);
}

const char* fa_get_error(void) { return g_err; }

void fa_set_wait_limit_ns(uint64_t ns) { g_wait_ns.store(ns > 0 ? ns : default_wait_ns()); }

void fa_debug_set_flags(int flags) { g_debug_flags.store(flags); }

const char* fa_version(void) { return "exact-io-aware-attention sm_100a 0.1"; }

}  // extern "C"

// ----------------------------------------------------------------------------- backward without allocation
// Some callers cannot allocate device memory: a plugin running inside another runtime that owns
// every byte of device memory and gives its plugins no workspace, or a latency-critical loop where
// the implicit device synchronisation of cudaMalloc is not acceptable.  fa_bwd_noalloc serves
// them: the backward's scratch (the fp32 dQ accumulator and D) lives in the fixed array below,
// which is part of the library image.  Every GPU that loads the library holds these bytes until
// the process exits.
namespace {

constexpr size_t kNoallocScratchBytes = size_t(48) << 20;   // 48 MiB
static __device__ __align__(256) unsigned char g_fa_noalloc_scratch[kNoallocScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {};

// The device address of the scratch array on the current device.  In host code the array's name
// is only a host-side stand-in, so the address is looked up once per device (with that device
// current) and cached.
fa_status noalloc_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(FA_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(FA_ERR_UNSUPPORTED, "device ordinal %d is out of range", dev);
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_fa_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr)
      return fail(FA_ERR_CUDA, "cudaGetSymbolAddress(static scratch): %s", cudaGetErrorString(e));
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return FA_OK;
}

}  // namespace

extern "C" {

fa_status fa_bwd_noalloc(const void* q, const void* k, const void* v, const void* o, const float* lse, const void* dO,
                         void* dq, void* dk, void* dv, int B, int H, int N, int d, float scale, int causal,
                         const int32_t* key_lens, float dropout_p, uint64_t seed, cudaStream_t stream) {
  const size_t need = fa_bwd_workspace_size(B, H, N, d);
  if (need > kNoallocScratchBytes)
    return fail(FA_ERR_INVALID_ARG,
                "fa_bwd_noalloc: B=%d H=%d N=%d d=%d needs %zu bytes of scratch, more than the library's "
                "static %zu bytes; call fa_bwd with a workspace instead",
                B, H, N, d, need, kNoallocScratchBytes);
  void* ws = nullptr;
  const fa_status st = noalloc_scratch(&ws);
  if (st != FA_OK) return st;
  return fa_bwd(q, k, v, o, lse, dO, dq, dk, dv, B, H, N, d, scale, causal, key_lens, dropout_p, seed, ws,
                kNoallocScratchBytes, stream);
}

size_t fa_bwd_noalloc_max_scratch(void) { return kNoallocScratchBytes; }

}  // extern "C"
