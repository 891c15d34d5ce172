// Exact attention backward for sm_100a, recomputing each probability block from Q, K and the
// saved per-row logsumexp instead of storing P ("48 FlashAttention", block "Tiling и online
// softmax", paragraph "Backward — тоже без N×N"; "Flash Attention：如何通过硬件感知优化重塑注意力机制的
// 未来", section 2.2: keep only the softmax normalisers and rebuild the attention weights on demand).  Gradients are the exact
// derivatives of O = dropout(softmax(mask(tau Q K^T))) V:
//   dV = Pt^T dO,  dPt = dO V^T,  dP = dPt * Z/(1-p),  D_i = rowsum(dO * O)_i,
//   dS = P * (dP - D),  dQ = tau dS K,  dK = tau dS^T Q.
//
// Three launches:
//   fa_bwd_prep_kernel    D = rowsum(dO * O) in fp32; clears the fp32 dQ accumulator and the work
//                         counter of the main launch
//   fa_bwd_sm100_kernel   persistent, one CTA per SM; work items (b, h, 128-key tile) with K and V
//                         resident, each looping over its query tiles; S^T, dP^T, dV, dK, dQ on
//                         tcgen05; dQ added into the fp32 accumulator with TMA bulk reductions (fp32
//                         gradient accumulation, as the mixed-precision advice in section 3.2 of the
//                         same blog post asks)
//   fa_bwd_dq_kernel      dQ = bf16(tau * accumulator)
//
// Main kernel roles (16 warps, four warpgroups with their own register budgets):
//   warps 0-7  compute, two warpgroups: thread r of warp w owns key row r (TMEM lane r) for the query
//              half w / 4 (64 query columns of each tile).  P^T = exp2(S^T tau log2e - lse2), masks,
//              dropout; (P*Z)^T as bf16 into TMEM over the half's first 32 score columns (dV takes
//              1/(1-p) at the end); dS^T = P^T (dP^T Z/(1-p) - D) as bf16 into TMEM over the dP^T
//              columns already read (the A operand of dK) and into a swizzled shared-memory tile (the
//              B operand of dQ^T); dV epilogue (half of the features each)
//   warps 8-11 dQ: read the dQ^T tile from TMEM (lane = feature, column = query), stage it in shared
//              memory and add it to the accumulator with TMA bulk reductions; dK epilogue; with
//              dropout, the keep bits of the tiles two ahead
//   warp 12    producer: takes the work items (item queue below), TMA K and V per item, Q (2 deep)
//              and dO (1 deep at D=128, 2 at D=64) per query tile
//   warp 13    MMA issuer; warp 14 loads -lse and -D per query tile into shared memory; warp 15 idle
// TMEM (512 columns): S^T [0,128), then (P*Z)^T; dP^T [128,256), then dS^T, then (D = 128) dQ^T;
// dV [256,256+D); dK [256+D,256+2D); at D = 64 dQ^T has columns of its own, [384,512).  MMA order per
// query tile t:
//   dV_t (per query half), S_{t+1}, dK_t (per query half), dQ^T_t, dP_{t+1}
// so S_{t+1} runs while the compute warps make dS_t, and dK_t reads dS^T before dQ^T_t overwrites it
// (MMAs of one thread execute in issue order).  At D = 128, dP_{t+1} waits until the dQ warps have
// read dQ^T_t out of the shared columns; at D = 64 only dQ^T_{t+1} waits for that.
#pragma once
#include <cuda_bf16.h>
#include "sm100.cuh"
#include "dropout_hash.cuh"

namespace fa {

struct BwdParams {  // (the main kernel also takes tensor maps of q, k, v, dO and the dQ accumulator)
  const __nv_bfloat16* o;      // [B,H,N,D]   (prep)
  const __nv_bfloat16* dO;     // [B,H,N,D]   (prep)
  const float* lse;            // [B,H,N]
  float* dvec;                 // [B,H,N]     D = rowsum(dO * O)
  float* dq_acc;               // [B,H,N,D]   fp32
  __nv_bfloat16* dq;           // [B,H,N,D]
  __nv_bfloat16* dk;           // [B,H,N,D]
  __nv_bfloat16* dv;           // [B,H,N,D]
  const int32_t* key_lens;     // [B] or null
  int B, H, N;
  int n_tiles;                 // ceil(N / 128)
  int causal;
  float scale;                 // tau
  float scale_log2;            // tau * log2(e)
  int dropout;
  uint32_t drop_thr;
  float drop_scale;
  uint64_t seed;
  uint64_t wait_ns;
  int out_align32;             // dk and dv are 32-byte aligned: epilogues use 32-byte stores
  int kt_major;                // 1-D grid in head groups, key-tile-major inside a group; else (n_tiles, B*H)
  int head_group;              // heads per group (kt_major)
  int debug_flags;             // bit 1: the producer never delivers the first Q tile (exercises the timeout path)
  unsigned int* work_ctr;      // items handed out beyond the first one of each CTA (zeroed by the prep kernel)
};

constexpr float kLog2e = 1.4426950408889634074f;

// ----------------------------------------------------------------------------- prep
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_prep_kernel(const BwdParams p) {
  constexpr int TPR = D / 8;                       // threads per row, 8 elements (16 bytes) each
  if (blockIdx.x == 0 && threadIdx.x == 0) *p.work_ctr = 0u;   // the main kernel's item counter
  const uint64_t rows = uint64_t(p.B) * p.H * p.N;
  const uint64_t t = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x;
  const uint64_t row = t / TPR;
  const int part = int(t % TPR);
  float acc = 0.f;
  if (row < rows) {
    const uint4 ov = reinterpret_cast<const uint4*>(p.o + row * D)[part];
    const uint4 gv = reinterpret_cast<const uint4*>(p.dO + row * D)[part];
    const __nv_bfloat162* o2 = reinterpret_cast<const __nv_bfloat162*>(&ov);
    const __nv_bfloat162* g2 = reinterpret_cast<const __nv_bfloat162*>(&gv);
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float2 a = __bfloat1622float2(o2[e]);
      const float2 c = __bfloat1622float2(g2[e]);
      acc = fmaf(a.x, c.x, acc);
      acc = fmaf(a.y, c.y, acc);
    }
    float4* z = reinterpret_cast<float4*>(p.dq_acc + row * D + part * 8);
    z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
    z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
#pragma unroll
  for (int off = TPR / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
  if (row < rows && part == 0) p.dvec[row] = acc;
}

// ----------------------------------------------------------------------------- dq convert
template <int D>
__global__ void __launch_bounds__(256) fa_bwd_dq_kernel(const BwdParams p) {
  const uint64_t n8 = uint64_t(p.B) * p.H * p.N * D / 8;
  for (uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n8; i += uint64_t(gridDim.x) * blockDim.x) {
    const float4 a = reinterpret_cast<const float4*>(p.dq_acc)[2 * i];
    const float4 c = reinterpret_cast<const float4*>(p.dq_acc)[2 * i + 1];
    uint4 r;
    r.x = pack_bf16x2(a.x * p.scale, a.y * p.scale);
    r.y = pack_bf16x2(a.z * p.scale, a.w * p.scale);
    r.z = pack_bf16x2(c.x * p.scale, c.y * p.scale);
    r.w = pack_bf16x2(c.z * p.scale, c.w * p.scale);
    reinterpret_cast<uint4*>(p.dq)[i] = r;
  }
}

// ----------------------------------------------------------------------------- main
template <int D, bool DROPOUT>
struct BwdLayout {
  static constexpr int TILE = 128 * D * 2;
  static constexpr int SUB = 128 * 128;
  static constexpr int QS = 2;                                  // Q ring (and per-tile statistics) depth
  static constexpr int DS = (D == 128) ? 1 : 2;                  // dO ring depth (dO_{t+1} is needed after dV_t)
  static constexpr int K_OFF = 0;
  static constexpr int V_OFF = K_OFF + TILE;
  static constexpr int Q_OFF = V_OFF + TILE;
  static constexpr int DO_OFF = Q_OFF + QS * TILE;
  static constexpr int DS_OFF = DO_OFF + DS * TILE;          // 128 keys x 128 queries bf16, 2 panels
  // dQ staging for the bulk reductions: per dQ warp, QPR queries x FPW features of fp32
  static constexpr int FPW = (D == 128) ? 32 : 16;            // dQ^T features per warp (TMEM lanes with data)
  static constexpr int STG_BYTES = (D == 128 && DROPOUT) ? 16384 : 32768;
  static constexpr int STAGE_BYTES = STG_BYTES / 4;
  static constexpr int QPR = STAGE_BYTES / (FPW * 4);          // queries per reduction round
  static constexpr int ROUNDS = 128 / QPR;
  static constexpr int STG_OFF = DS_OFF + 2 * SUB;
  static constexpr int KEEP_OFF = STG_OFF + STG_BYTES;       // dropout keep bits: 2 stages x 128 keys x 128 bits
  static constexpr int STAT_OFF = KEEP_OFF + (DROPOUT ? 2 * 128 * 16 : 0);   // per stage: -lse2[128], -D[128]
  static constexpr int NQI = 8;                               // item queue depth
  static constexpr int ITEM_OFF = STAT_OFF + QS * 1024;       // item ids, int32 [NQI]
  static constexpr int BAR_OFF = ITEM_OFF + NQI * 4;
  // kv_full, q_full[QS], q_empty[QS], stat_full[QS], do_full[DS], do_empty[DS], s_full, dp_full,
  // p_full[2], ds_full[2], dq_full, dq_empty, ds_free, fin, keep_full[2], kv_empty, dk_free,
  // item_full[NQI], item_empty[NQI], keep_empty[2]
  static constexpr int NBARS = 1 + 3 * QS + 2 * DS + 10 + 2 + 2 + 2 * NQI + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  // TMEM: S^T, then (P*Z)^T over [0,64); dP^T, then dS^T over [128,192), then dQ^T; dV; dK
  static constexpr int ST_COL = 0, DPT_COL = 128, DV_COL = 256, DK_COL = 256 + D;
  // dQ^T: at D = 64 in columns of its own [384, 512), so that dP_{t+1} need not wait until the dQ
  // warps have read dQ^T_t out of the dP^T columns (only dQ^T_{t+1} waits for that); at D = 128 the
  // 512 columns are taken and dQ^T goes over dP^T/dS^T
  static constexpr int DQT_COL = (D == 64) ? 256 + 2 * D : DPT_COL;
  static constexpr bool DQT_OWN = DQT_COL != DPT_COL;
  static constexpr int TMEM_COLS = 512;
  static_assert(DK_COL + D <= TMEM_COLS, "TMEM budget");
  static_assert(BYTES <= 232448, "shared memory budget");
};

// 32 fp32 values of one row, scaled and rounded to bf16, stored as 64 bytes (two 32-byte stores
// when the destination allows it, else four 16-byte stores).
__device__ __forceinline__ void store_row32(__nv_bfloat16* dst, const uint32_t (&v)[32], float s, int align32) {
  uint32_t w[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) w[e] = pack_bf16x2(__uint_as_float(v[2 * e]) * s, __uint_as_float(v[2 * e + 1]) * s);
  if (align32) {
    st_global_v8(dst, w[0], w[1], w[2], w[3], w[4], w[5], w[6], w[7]);
    st_global_v8(dst + 16, w[8], w[9], w[10], w[11], w[12], w[13], w[14], w[15]);
  } else {
    uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
    for (int e = 0; e < 4; ++e) d4[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
  }
}

__device__ __forceinline__ bool warp_wait(uint64_t* bar, uint32_t parity, const WaitCtl& w) {
  return __all_sync(0xffffffffu, mbar_wait(bar, parity, w));
}

// Bulk tensor reduction (add) of a shared-memory box into global memory; no multicast.
__device__ __forceinline__ void tma_reduce_add_3d(const CUtensorMap* map, const void* src, int x, int y, int z) {
  asm volatile("cp.reduce.async.bulk.tensor.3d.global.shared::cta.add.bulk_group [%0, {%2, %3, %4}], [%1];"
               :: "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(x), "r"(y), "r"(z) : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

// Keep bits of the 128 query columns of tile `qrow0` for key k0 + r, made together by the four
// lanes that hold keys k0 + 4m .. k0 + 4m + 3 (m = r >> 2; r & 3 = lane & 3): lane s = r & 3 takes
// the draws of queries qrow0 + 4t + s (t = 0..31), each deciding the group's four keys, and a 4 x 4
// exchange of 32-bit words gives every lane its own key's bits.  Every lane of the warp calls it.
// Layout of the result: query column c of the tile, c = 64 qh + c', is bit
// 16 (c' & 1) + (c' >> 2) of word 2 qh + ((c' >> 1) & 1); keep_bit() reads it.
__device__ __forceinline__ uint4 keep_bits_row(const BwdParams& p, uint64_t row_base, int qrow0, int k0, int r) {
  const uint32_t s = uint32_t(r) & 3u;
  const uint64_t W = dropout_row_draws(p.N);
  uint64_t z = dropout_z(p.seed, (row_base + uint64_t(qrow0) + s) * W + uint64_t((k0 >> 2) + (r >> 2)));
  const uint64_t step = 4ull * W * kDropGamma;   // four queries on
  const uint32_t c = dropout_lane_c(p.drop_thr);
  // acc[hf]: keys 0 (bits 0-15) and 1 (bits 16-31) for t = 16 hf + bit; acc[2 + hf]: keys 2 and 3
  uint32_t acc[4];
#pragma unroll
  for (int hf = 0; hf < 2; ++hf) {
    uint32_t x01 = 0u, x23 = 0u;
#pragma unroll 4
    for (int tt = 0; tt < 16; ++tt) {
      const uint64_t x = dropout_mix(z);
      z += step;
      x01 |= ((dropout_flags(uint32_t(x), c) >> 15) & 0x00010001u) << tt;
      x23 |= ((dropout_flags(uint32_t(x >> 32), c) >> 15) & 0x00010001u) << tt;
    }
    acc[hf] = x01;
    acc[2 + hf] = x23;
  }
  // v[kk]: key kk's bits for queries 4t + s, bit t
  uint32_t v[4];
  v[0] = __byte_perm(acc[0], acc[1], 0x5410);
  v[1] = __byte_perm(acc[0], acc[1], 0x7632);
  v[2] = __byte_perm(acc[2], acc[3], 0x5410);
  v[3] = __byte_perm(acc[2], acc[3], 0x7632);
  auto pick = [&](uint32_t i) { return (i & 2u) ? ((i & 1u) ? v[3] : v[2]) : ((i & 1u) ? v[1] : v[0]); };
  // u[j] = lane j's word for this lane's key (queries 4t + j)
  uint32_t rr[4];
  rr[0] = pick(s);
#pragma unroll
  for (int d = 1; d < 4; ++d) rr[d] = __shfl_xor_sync(0xffffffffu, pick(s ^ uint32_t(d)), d);
  auto from = [&](uint32_t j) {   // u[j] = rr[j ^ s]
    const uint32_t i = j ^ s;
    return (i & 2u) ? ((i & 1u) ? rr[3] : rr[2]) : ((i & 1u) ? rr[1] : rr[0]);
  };
  const uint32_t u0 = from(0), u1 = from(1), u2 = from(2), u3 = from(3);
  return make_uint4(__byte_perm(u0, u1, 0x5410), __byte_perm(u2, u3, 0x5410), __byte_perm(u0, u1, 0x7632),
                    __byte_perm(u2, u3, 0x7632));
}
// The keep bit of query column c' (0..63) of a half from that half's two words.
__device__ __forceinline__ uint32_t keep_bit(const uint32_t (&kb)[2], int c) {
  return (kb[(c >> 1) & 1] >> (16 * (c & 1) + (c >> 2))) & 1u;
}

// Register split per warpgroup (launch: 512 threads x 128 = 65536 registers):
// 128 x (144 + 144 + 152 + 72) = 65536.
constexpr int kBwdThreads = 512;
constexpr int kBwdLaunchRegs = 128;   // the host checks the kernel's register count against this

// One work item: the 128-key tile kt of head bh, and the query tiles it meets.
struct BwdItem {
  int kt, bh, k0, kv_end, q_first, n_iter;
  uint64_t row_base;
};

// Item L of the launch order.  kt_major: groups of head_group heads one after another, key-tile-major
// inside a group (each head's heaviest causal key tiles start with its group); else head-major.
__device__ __forceinline__ BwdItem bwd_item(const BwdParams& p, int L) {
  BwdItem it;
  if (p.kt_major) {
    const int BH = p.B * p.H, G = p.head_group, per_group = G * p.n_tiles;
    const int g = L / per_group, r = L % per_group, gs = min(G, BH - g * G);
    it.kt = r / gs;
    it.bh = g * G + r % gs;
  } else {
    it.kt = L % p.n_tiles;
    it.bh = L / p.n_tiles;
  }
  it.k0 = it.kt * 128;
  it.kv_end = p.N;
  if (p.key_lens != nullptr) it.kv_end = min(it.kv_end, max(p.key_lens[it.bh / p.H], 0));
  it.q_first = p.causal ? it.kt : 0;
  it.n_iter = (it.k0 < it.kv_end) ? (p.n_tiles - it.q_first) : 0;
  it.row_base = uint64_t(it.bh) * uint64_t(p.N);
  return it;
}

// The item queue of a CTA: the producer warp takes items from the launch order, its first item
// statically (item blockIdx.x) and the rest from a global counter as it gets to them, and passes
// the ids of items that have query tiles to the other roles through a ring in shared memory (-1
// ends the sequence).  Consumers release a slot as soon as they have read it.
struct ItemQueue {
  volatile int* ids;       // [NQI]
  uint64_t* full;          // [NQI], one arrival (the producer)
  uint64_t* empty;         // [NQI], one arrival per consumer warp
  int nq;
  // the n-th id of the sequence (a bounded wait for the producer to post it); false on abort
  __device__ __forceinline__ bool peek(int n, int& id, const WaitCtl& wc) const {
    if (!__all_sync(0xffffffffu, mbar_wait(&full[n % nq], (n / nq) & 1, wc))) return false;
    id = ids[n % nq];
    return true;
  }
  __device__ __forceinline__ void release(int n, int lane) const {
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[n % nq]);
  }
};

// Walks the query tiles of the queued items, ahead of the current one: the dQ warps use it to make
// the dropout keep bits of the tiles two ahead, which may belong to the next item(s).
struct BwdTileCursor {
  int n, t;                // queue index and tile of the cursor
  BwdItem it;
  bool valid;
  __device__ __forceinline__ bool load(const BwdParams& p, const ItemQueue& q, const WaitCtl& wc) {
    int id;
    if (!q.peek(n, id, wc)) return false;
    valid = id >= 0;
    if (valid) it = bwd_item(p, id);
    return true;
  }
  __device__ __forceinline__ bool start(const BwdParams& p, const ItemQueue& q, const WaitCtl& wc) {
    n = 0;
    t = 0;
    return load(p, q, wc);
  }
  __device__ __forceinline__ bool advance(const BwdParams& p, const ItemQueue& q, const WaitCtl& wc) {
    if (!valid) return true;
    if (++t < it.n_iter) return true;
    t = 0;
    ++n;
    return load(p, q, wc);
  }
};

// Persistent: one CTA per SM, each taking items from the item queue above (dynamically balanced:
// a CTA takes the next item of the launch order when it gets to it).  TMEM is allocated and the
// barriers are set up once; every barrier phase counts tiles (g) or items (gi) over the whole
// sequence, so the Q/dO rings, the statistics and the keep bits run on from one item into the next:
// the next item's first Q and dO tiles load while the previous one finishes, and its K/V load as soon
// as the previous item's last MMA has read K and V.
// DQ: the kernel also forms dQ^T per tile and adds it into the fp32 accumulator (the fused path);
// without it (the separate-pass path, fa_bwd_split) it makes dK and dV only, and dS stays in TMEM.
template <int D, bool DROPOUT, bool DQ>
__global__ void __launch_bounds__(kBwdThreads, 1)
fa_bwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    const __grid_constant__ CUtensorMap tm_dq, const BwdParams p) {
  using L = BwdLayout<D, DROPOUT>;
  constexpr int QS = L::QS, DS = L::DS;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((smem_u32(smem) & 1023u) != 0) {
    if (tid == 0) record_status(kStatusBadSmemAlign);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* kv_full = bars;
  uint64_t* q_full = bars + 1;
  uint64_t* q_empty = q_full + QS;
  uint64_t* stat_full = q_empty + QS;
  uint64_t* do_full = stat_full + QS;
  uint64_t* do_empty = do_full + DS;
  uint64_t* s_full = do_empty + DS;
  uint64_t* dp_full = s_full + 1;
  uint64_t* p_full = dp_full + 1;     // [2]: query half
  uint64_t* ds_full = p_full + 2;     // [2]: query half
  uint64_t* dq_full = ds_full + 2;
  uint64_t* dq_empty = dq_full + 1;
  uint64_t* ds_free = dq_empty + 1;
  uint64_t* fin = ds_free + 1;        // per item: its last MMA has completed
  uint64_t* keep_full = fin + 1;      // [2]: stage
  uint64_t* kv_empty = keep_full + 2; // per item: K and V may be replaced
  uint64_t* dk_free = kv_empty + 1;   // per item: the dK epilogue has read the accumulator
  const ItemQueue queue{reinterpret_cast<volatile int*>(smem + L::ITEM_OFF), dk_free + 1, dk_free + 1 + L::NQI, L::NQI};
  // [2]: stage; the compute warps have read the keep bits of the stage's tile (used without DQ,
  // where no dQ^T MMA orders the keep-bit warps behind the compute warps)
  uint64_t* keep_empty = dk_free + 1 + 2 * L::NQI;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);
  float* stat = reinterpret_cast<float*>(smem + L::STAT_OFF);
  uint4* keep_smem = reinterpret_cast<uint4*>(smem + L::KEEP_OFF);   // [2][128]

  const int G = int(gridDim.x), cta = int(blockIdx.x);
  const int n_items = p.B * p.H * p.n_tiles;

  if (tid == 0) {
    mbar_init(kv_full, 1);
    for (int s = 0; s < QS; ++s) {
      mbar_init(&q_full[s], 1);
      mbar_init(&q_empty[s], 1);
      mbar_init(&stat_full[s], 32);
    }
    for (int s = 0; s < DS; ++s) {
      mbar_init(&do_full[s], 1);
      mbar_init(&do_empty[s], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(dp_full, 1);
    for (int h = 0; h < 2; ++h) {
      mbar_init(&p_full[h], 4);
      mbar_init(&ds_full[h], 4);
      mbar_init(&keep_full[h], 4);
      mbar_init(&keep_empty[h], 8);
    }
    mbar_init(dq_full, 1);
    mbar_init(dq_empty, 4);
    mbar_init(ds_free, 1);
    mbar_init(fin, 1);
    mbar_init(kv_empty, 1);
    mbar_init(dk_free, 4);
    for (int i = 0; i < L::NQI; ++i) {
      mbar_init(&queue.full[i], 1);
      mbar_init(&queue.empty[i], 14);   // stats, MMA, 8 compute and 4 dQ warps
    }
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 13) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{p.wait_ns, abort_flag};

  if (warp == 15) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 72;\n" ::: "memory");
  } else if (warp == 14) {
    // =========================================================== per-tile statistics
    asm volatile("setmaxnreg.dec.sync.aligned.u32 72;\n" ::: "memory");
    int g = 0;   // query tiles so far (all items)
    bool ok = true;
    for (int n = 0; ok; ++n) {
      int id;
      if (!queue.peek(n, id, wc)) break;
      queue.release(n, lane);
      if (id < 0) break;
      const BwdItem it = bwd_item(p, id);
      for (int t = 0; t < it.n_iter; ++t, ++g) {
        const int sq = g % QS;
        const int qrow0 = (it.q_first + t) * 128;
        // the stage is reused once dK of tile g-QS (after every read of its statistics) is done
        if (g >= QS && !warp_wait(&q_empty[sq], ((g / QS) - 1) & 1, wc)) { ok = false; break; }
        // negated: -lse in the exp2 domain and -D; one 16-byte store per lane and array
        float* st_l = stat + sq * 256;
        float lv[4], dv[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int q = qrow0 + lane * 4 + e;
          lv[e] = q < p.N ? -p.lse[it.row_base + q] * kLog2e : 0.f;
          dv[e] = q < p.N ? -p.dvec[it.row_base + q] : 0.f;
        }
        reinterpret_cast<float4*>(st_l)[lane] = make_float4(lv[0], lv[1], lv[2], lv[3]);
        reinterpret_cast<float4*>(st_l + 128)[lane] = make_float4(dv[0], dv[1], dv[2], dv[3]);
        mbar_arrive(&stat_full[sq]);
      }
    }
  } else if (warp == 12) {
    // =========================================================== producer
    asm volatile("setmaxnreg.dec.sync.aligned.u32 72;\n" ::: "memory");
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      prefetch_tmap(&tm_do);
      prefetch_tmap(&tm_dq);
    }
    int g = 0, gi = 0;           // query tiles and items with tiles so far
    int issued_q = 0, issued_do = 0;
    bool ok = true;
    auto load_q_do = [&](const BwdItem& it, int t) -> bool {   // tile t of item it, global tile g
      const int sq = g % QS, sd = g % DS;
      const int qrow0 = (it.q_first + t) * 128;
      if (g >= QS && !warp_wait(&q_empty[sq], ((g / QS) - 1) & 1, wc)) return false;
      if (g == 0 && (p.debug_flags & 2)) return false;   // test hook: the first Q tile never arrives
      if (lane == 0) {
        mbar_arrive_expect_tx(&q_full[sq], L::TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::Q_OFF + sq * L::TILE + c * L::SUB, &tm_q, &q_full[sq], c * 64, qrow0, it.bh);
      }
      issued_q = g + 1;
      if (g >= DS && !warp_wait(&do_empty[sd], ((g / DS) - 1) & 1, wc)) return false;
      if (lane == 0) {
        mbar_arrive_expect_tx(&do_full[sd], L::TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::DO_OFF + sd * L::TILE + c * L::SUB, &tm_do, &do_full[sd], c * 64, qrow0, it.bh);
      }
      issued_do = g + 1;
      ++g;
      return true;
    };
    int n_posted = 0;   // ids posted to the item queue
    auto post = [&](int id) -> bool {
      if (n_posted >= L::NQI && !warp_wait(&queue.empty[n_posted % L::NQI], ((n_posted / L::NQI) - 1) & 1, wc))
        return false;
      if (lane == 0) {
        queue.ids[n_posted % L::NQI] = id;
        mbar_arrive(&queue.full[n_posted % L::NQI]);
      }
      __syncwarp();
      ++n_posted;
      return true;
    };
    for (int taken = 0; ok; ++taken) {
      int id = cta;
      if (taken > 0) {
        unsigned int c = 0;
        if (lane == 0) c = atomicAdd(p.work_ctr, 1u);
        id = G + int(__shfl_sync(0xffffffffu, c, 0));
      }
      if (id >= n_items) break;
      const BwdItem it = bwd_item(p, id);
      if (it.n_iter == 0) {
        // a key tile past the key length: no gradient flows into it, its dK and dV rows are zero
        for (int e = lane; e < 128 * (D / 8); e += 32) {
          const int row = it.k0 + e / (D / 8), c = e % (D / 8);
          if (row < p.N) {
            reinterpret_cast<uint4*>(p.dk + (it.row_base + row) * D)[c] = make_uint4(0, 0, 0, 0);
            reinterpret_cast<uint4*>(p.dv + (it.row_base + row) * D)[c] = make_uint4(0, 0, 0, 0);
          }
        }
        continue;
      }
      if (!post(id)) { ok = false; break; }
      // the item's first Q and dO tiles need only ring slots: load them before waiting for K/V
      if (!load_q_do(it, 0)) { ok = false; break; }
      // K and V replace the previous item's once its last MMA has read them
      if (gi >= 1 && !warp_wait(kv_empty, (gi - 1) & 1, wc)) { ok = false; break; }
      if (lane == 0) {
        mbar_arrive_expect_tx(kv_full, 2 * L::TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c) {
          tma_load_3d(smem + L::K_OFF + c * L::SUB, &tm_k, kv_full, c * 64, it.k0, it.bh);
          tma_load_3d(smem + L::V_OFF + c * L::SUB, &tm_v, kv_full, c * 64, it.k0, it.bh);
        }
      }
      ++gi;
      for (int t = 1; t < it.n_iter; ++t)
        if (!load_q_do(it, t)) { ok = false; break; }
    }
    if (ok) post(-1);   // end of the sequence
    // every copy started here lands before the CTA releases its shared memory
    if (lane == 0) {
      if (gi >= 1) mbar_drain(kv_full, (gi - 1) & 1, p.wait_ns);
      for (int t = max(0, issued_q - QS); t < issued_q; ++t) mbar_drain(&q_full[t % QS], (t / QS) & 1, p.wait_ns);
      for (int t = max(0, issued_do - DS); t < issued_do; ++t) mbar_drain(&do_full[t % DS], (t / DS) & 1, p.wait_ns);
    }
    __syncwarp();
  } else if (warp == 13) {
    // =========================================================== MMA issuer
    // The whole warp runs the loop (descriptors stay warp-uniform); the lane that elect.sync picks
    // issues every MMA and commit, so one thread owns all tcgen05 work, and the MMAs execute in
    // issue order: an MMA that overwrites TMEM columns runs after every earlier MMA that reads them.
    asm volatile("setmaxnreg.dec.sync.aligned.u32 72;\n" ::: "memory");
    constexpr uint32_t kIdS = idesc_bf16(128, 128, false, false);   // K (V) and Q (dO) K-major
    constexpr uint32_t kIdG = idesc_bf16(128, D, false, true);      // dV, dK: A in TMEM, B MN-major
    constexpr uint32_t kIdQ = idesc_bf16(D, 128, true, true);       // dQ^T: K^T, dS^T both MN-major
    // descriptors: low word = s0 + (byte offset in shared memory >> 4) + leading-offset field
    // (K-major: 16; MN-major: one 64-column panel)
    const uint32_t s0 = smem_u32(smem) >> 4;
    constexpr uint32_t kHi = sdesc_sw128_hi(1024), kKM = sdesc_lbo(16), kMN = sdesc_lbo(L::SUB);
    auto lo = [&](int off, uint32_t lbo) { return s0 + uint32_t(off >> 4) + lbo; };
    auto issue_s = [&](int g) {   // S^T = K Q_g^T  (M = 128 keys, N = 128 queries, K = D)
      const uint32_t k_lo = lo(L::K_OFF, kKM), q_lo = lo(L::Q_OFF + (g % QS) * L::TILE, kKM);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk >> 2) * L::SUB + (kk & 3) * 32) >> 4;
        mma_ss_elect(tmem + L::ST_COL, sdesc_join(k_lo + off, kHi), sdesc_join(q_lo + off, kHi), kIdS,
                    kk > 0 ? 1u : 0u);
      }
      mma_commit_elect(s_full);
    };
    auto issue_dp = [&](int g) {   // dP^T = V dO_g^T
      const uint32_t v_lo = lo(L::V_OFF, kKM), do_lo = lo(L::DO_OFF + (g % DS) * L::TILE, kKM);
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk >> 2) * L::SUB + (kk & 3) * 32) >> 4;
        mma_ss_elect(tmem + L::DPT_COL, sdesc_join(v_lo + off, kHi), sdesc_join(do_lo + off, kHi), kIdS,
                    kk > 0 ? 1u : 0u);
      }
      mma_commit_elect(dp_full);
    };
    auto wait = [&](uint64_t* bar, uint32_t parity) { return warp_wait(bar, parity, wc); };
    int g = 0, gi = 0;
    bool ok = true;
    for (int n = 0; ok; ++n) {
      int id;
      if (!queue.peek(n, id, wc)) { ok = false; break; }
      queue.release(n, lane);
      if (id < 0) break;
      const BwdItem it = bwd_item(p, id);
      if (!wait(kv_full, gi & 1)) { ok = false; break; }
      // first S and dP of the item; dP overwrites the columns where the previous tile's dQ^T sat
      if (!wait(&q_full[g % QS], (g / QS) & 1)) { ok = false; break; }
      tc_fence_after();
      issue_s(g);
      if (DQ && !L::DQT_OWN && g >= 1 && !wait(dq_empty, (g - 1) & 1)) { ok = false; break; }
      if (!wait(&do_full[g % DS], (g / DS) & 1)) { ok = false; break; }
      tc_fence_after();
      issue_dp(g);
      for (int t = 0; t < it.n_iter; ++t, ++g) {
        const bool more = t + 1 < it.n_iter;
        const uint32_t acc0 = t > 0 ? 1u : 0u;
        // dV += (P*Z)^T dO_g, query half by query half (A = (P*Z)^T in TMEM: half h packed at
        // columns [64h, 64h+32); B = dO MN-major: N = D, K = 16 queries per step).  The compute
        // warps give P of an item's first tile only after their dV epilogue of the previous item.
        {
          const uint32_t do_lo = lo(L::DO_OFF + (g % DS) * L::TILE, kMN);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (!wait(&p_full[h], g & 1)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int kk = 4 * h; kk < 4 * h + 4; ++kk)
              mma_ts_elect(tmem + L::DV_COL, tmem + L::ST_COL + 64 * h + (kk & 3) * 8,
                          sdesc_join(do_lo + kk * (2048 >> 4), kHi), kIdG, kk > 0 ? 1u : acc0);
          }
          if (!ok) break;
        }
        mma_commit_elect(&do_empty[g % DS]);   // dO_g: last read by dV_g
        // S_{g+1} over the (P*Z)^T that dV_g has just been given
        if (more) {
          if (!wait(&q_full[(g + 1) % QS], ((g + 1) / QS) & 1)) { ok = false; break; }
          tc_fence_after();
          issue_s(g + 1);
        }
        // the first dK of an item overwrites the accumulator: the previous item's dK epilogue must
        // have read it
        if (t == 0 && gi >= 1 && !wait(dk_free, (gi - 1) & 1)) { ok = false; break; }
        // dK += dS^T Q_g, query half by query half (A = dS^T in TMEM over the dP^T columns, half h
        // packed at [128 + 64h, 128 + 64h + 32); B = Q MN-major)
        {
          const uint32_t q_lo = lo(L::Q_OFF + (g % QS) * L::TILE, kMN);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (!wait(&ds_full[h], g & 1)) { ok = false; break; }
            tc_fence_after();
#pragma unroll
            for (int kk = 4 * h; kk < 4 * h + 4; ++kk)
              mma_ts_elect(tmem + L::DK_COL, tmem + L::DPT_COL + 64 * h + (kk & 3) * 8,
                          sdesc_join(q_lo + kk * (2048 >> 4), kHi), kIdG, kk > 0 ? 1u : acc0);
          }
          if (!ok) break;
        }
        mma_commit_elect(&q_empty[g % QS]);    // Q_g: last read by dK_g
        if (DQ) {
          // dQ^T = K^T dS^T (M = D, N = 128 queries, K = 128 keys; B = dS^T from shared memory):
          // over the dS^T/dP^T columns after dK_g has read them, or in its own columns once the dQ
          // warps have read the previous tile's
          if (L::DQT_OWN && g >= 1 && !wait(dq_empty, (g - 1) & 1)) { ok = false; break; }
          const uint32_t k_lo = lo(L::K_OFF, kMN), ds_lo = lo(L::DS_OFF, kMN);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss_elect(tmem + L::DQT_COL, sdesc_join(k_lo + kk * (2048 >> 4), kHi),
                        sdesc_join(ds_lo + kk * (2048 >> 4), kHi), kIdQ, kk > 0 ? 1u : 0u);
          mma_commit_elect(dq_full);
          mma_commit_elect(ds_free);             // the shared-memory dS tile is free again
        }
        // dP_{g+1} once the dQ warps have read dQ^T out of those columns (with DQ; without it, the
        // dK MMAs issued above read dS^T there first: MMAs run in issue order)
        if (more) {
          if (DQ && !L::DQT_OWN && !wait(dq_empty, g & 1)) { ok = false; break; }
          if (!wait(&do_full[(g + 1) % DS], ((g + 1) / DS) & 1)) { ok = false; break; }
          tc_fence_after();
          issue_dp(g + 1);
        }
      }
      if (!ok) break;
      mma_commit_elect(fin);        // the item's dV and dK are complete
      mma_commit_elect(kv_empty);   // and K, V are no longer read
      ++gi;
    }
    // every MMA issued above completes before TMEM is released: wait for the last item's fin (on
    // an abort, commit once more and wait for that)
    if (!ok) mma_commit_elect(fin);
    if (lane == 0 && (gi >= 1 || !ok)) mbar_drain(fin, ok ? ((gi - 1) & 1) : (gi & 1), p.wait_ns);
    __syncwarp();
  } else if (warp < 8) {
    // =========================================================== compute (key row r, query half qh)
    asm volatile("setmaxnreg.inc.sync.aligned.u32 144;\n" ::: "memory");
    const int qh = warp >> 2;                 // query columns [64 qh, 64 qh + 64) of every tile
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
    const float sl2 = p.scale_log2;
    bool ok = true;
    uint8_t* ds_smem = smem + L::DS_OFF + qh * L::SUB;   // this half's 64 query columns: one panel
    int g = 0, gi = 0;   // query tiles and items with tiles so far (barrier phases)
    for (int n = 0; ok; ++n) {   // items of the queue
    int id;
    if (!queue.peek(n, id, wc)) { ok = false; break; }
    queue.release(n, lane);
    if (id < 0) break;
    const BwdItem itm = bwd_item(p, id);
    const int kt = itm.kt, k0 = itm.k0, kv_end = itm.kv_end, q_first = itm.q_first, n_iter = itm.n_iter;
    const uint64_t row_base = itm.row_base;
    const int key = k0 + r;
    for (int t = 0; t < n_iter; ++t, ++g) {   // (body indented one level less than the loop above)
      const int sq = g % QS;
      const int qrow0 = (q_first + t) * 128;
      const int qc0 = qrow0 + 64 * qh;         // first query of this half
      const float* st_l = stat + sq * 256 + 64 * qh;
      const bool need_mask = (k0 + 128 > kv_end) || (qc0 + 64 > p.N) || (p.causal && q_first + t == kt);
      uint32_t kb[2] = {0u, 0u};   // dropout keep bits of this key row and query half (keep_bit)
      if (DROPOUT) {
        if (!warp_wait(&keep_full[g & 1], (g >> 1) & 1, wc)) { ok = false; break; }
        const uint2 w = reinterpret_cast<const uint2*>(&keep_smem[(g & 1) * 128 + r])[qh];
        kb[0] = w.x;
        kb[1] = w.y;
      }
      if (!warp_wait(s_full, g & 1, wc)) { ok = false; break; }
      if (!warp_wait(&stat_full[sq], (g / QS) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      // ---- P^T = exp2(S^T tau log2e - lse2) over this half's 64 query columns
      float pr[64];
      {
        uint32_t* sr = reinterpret_cast<uint32_t*>(pr);
        tmem_ld32(lane_base + L::ST_COL + 64 * qh, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(lane_base + L::ST_COL + 64 * qh + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld_wait();
        reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      }
      {
        const uint64_t sl2x2 = f2_make(sl2, sl2);
        // -lse2 of four query columns per 16-byte (broadcast) load
        const float4* nl4 = reinterpret_cast<const float4*>(st_l);
#pragma unroll
        for (int c = 0; c < 64; c += 4) {
          const float4 nl = nl4[c >> 2];
          float x0, x1, x2, x3;
          f2_split(f2_fma(f2_make(pr[c], pr[c + 1]), sl2x2, f2_make(nl.x, nl.y)), x0, x1);
          f2_split(f2_fma(f2_make(pr[c + 2], pr[c + 3]), sl2x2, f2_make(nl.z, nl.w)), x2, x3);
          pr[c] = ex2_approx(x0);
          pr[c + 1] = ex2_approx(x1);
          pr[c + 2] = ex2_approx(x2);
          pr[c + 3] = ex2_approx(x3);
        }
      }
      if (need_mask) {
        // allowed: key < kv_end, query < N, and (not causal or key <= query)
        const int lim_q = p.N - qc0;                                    // columns < lim_q exist
        const int from_q = p.causal ? key - qc0 : -1;                   // causal: columns >= from_q
        const bool key_ok = key < kv_end;
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (!key_ok || c >= lim_q || c < from_q) pr[c] = 0.f;
      }
      {
        uint32_t pk[32];
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          float a = pr[2 * e], bb = pr[2 * e + 1];
          if (DROPOUT) {   // P * Z; dV takes the 1/(1-p) factor in its fp32 epilogue
            a = keep_bit(kb, 2 * e) ? a : 0.f;
            bb = keep_bit(kb, 2 * e + 1) ? bb : 0.f;
          }
          pk[e] = pack_bf16x2(a, bb);
        }
        // (P*Z)^T over the first 32 of this half's score columns, already read
        tmem_st32(lane_base + L::ST_COL + 64 * qh, pk);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[qh]);

      // ---- dS^T = P^T * (dP^T Z/(1-p) - D), in chunks of 32 query columns; written twice: as bf16
      // pairs into TMEM over the dP^T columns already read (the A operand of dK) and into this
      // half's shared-memory panel (the B operand of dQ^T)
      if (!warp_wait(dp_full, g & 1, wc)) { ok = false; break; }
      // the shared-memory dS tile is free: dQ^T of the previous tile has read it
      if (DQ && g >= 1 && !warp_wait(ds_free, (g - 1) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      if (DROPOUT) {
        // The keep bits again, through a volatile read: otherwise the compiler keeps the per-column
        // keep predicates of the P phase alive across the dP wait, which costs registers (spills).
        const volatile uint32_t* kv =
            reinterpret_cast<const volatile uint32_t*>(&keep_smem[(g & 1) * 128 + r]) + 2 * qh;
        kb[0] = kv[0];
        kb[1] = kv[1];
      }
#pragma unroll
      for (int cc = 0; cc < 2; ++cc) {
        uint32_t dr[32];
        tmem_ld32(lane_base + L::DPT_COL + 64 * qh + 32 * cc, dr);
        tmem_ld_wait();
        reg_fence32(dr);
        uint32_t pk[16];
        const float4* nd4 = reinterpret_cast<const float4*>(st_l + 128);   // -D, four columns per load
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int c = 32 * cc + 2 * e;
          const float4 nd = nd4[c >> 2];
          float dpa = __uint_as_float(dr[2 * e]), dpb = __uint_as_float(dr[2 * e + 1]);
          if (DROPOUT) {
            dpa = keep_bit(kb, c) ? dpa * p.drop_scale : 0.f;
            dpb = keep_bit(kb, c + 1) ? dpb * p.drop_scale : 0.f;
          }
          float da, db;   // dS = P (dP - D), as P * (dP + (-D)) on pairs
          const uint64_t nd2 = (e & 1) ? f2_make(nd.z, nd.w) : f2_make(nd.x, nd.y);
          f2_split(f2_mul(f2_make(pr[c], pr[c + 1]), f2_add(f2_make(dpa, dpb), nd2)), da, db);
          pk[e] = pack_bf16x2(da, db);
        }
        tmem_st16(lane_base + L::DPT_COL + 64 * qh + 16 * cc, pk);
        // dS (queries contiguous) into the 128-byte-swizzled panel: row = key r, 16-byte chunks of 8
        if (DQ) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int chunk = 4 * cc + u;
            uint4* dst = reinterpret_cast<uint4*>(ds_smem + r * 128 + ((chunk ^ (r & 7)) << 4));
            *dst = make_uint4(pk[4 * u], pk[4 * u + 1], pk[4 * u + 2], pk[4 * u + 3]);
          }
        }
      }
      if (DQ) fence_proxy_async_smem();   // generic-proxy stores -> visible to the tensor core
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&ds_full[qh]);
      if (!DQ && DROPOUT && lane == 0) mbar_arrive(&keep_empty[g & 1]);   // its keep bits are read
    }
    if (!ok) break;
    // ---- dV epilogue: this half of the feature columns
    constexpr int HD = D / 2;
    if (!warp_wait(fin, gi & 1, wc)) { ok = false; break; }
    ++gi;
    tc_fence_after();
    {
      const float s = DROPOUT ? p.drop_scale : 1.f;
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {
        uint32_t vr[32];
        tmem_ld32(lane_base + L::DV_COL + qh * HD + c * 32, vr);
        tmem_ld_wait();
        reg_fence32(vr);
        if (key < p.N) store_row32(p.dv + (row_base + key) * D + qh * HD + c * 32, vr, s, p.out_align32);
      }
    }
    // the next item's first dV MMA (which overwrites the accumulator) waits for this warp's next
    // P arrival, which comes after these reads
    tc_fence_before();
    }
  } else {
    // =========================================================== dQ + dK epilogue (warps 8-11)
    // TMEM holds dQ^T in the dP^T columns: lane = feature, column = query.  D=128: feature
    // 32*quarter + lane; D=64 (M=64 layout): feature 16*quarter + lane on lanes 0-15.  Each warp
    // stages its features for QPR queries in its slice of the staging buffer ([query][feature],
    // fp32) and adds that box to the accumulator with one TMA bulk reduction; the reductions run
    // in the background while the next tiles are computed.  (A red.global.add per element was
    // measured 25 % slower on the headline backward: the L2 resolves whole-line bulk reductions
    // faster than word-sized ones.)  With dropout these warps also make the keep bits of the tiles
    // ahead (two stages in shared memory), so that the compute warps only read them.
    asm volatile("setmaxnreg.inc.sync.aligned.u32 152;\n" ::: "memory");
    const int quarter = warp - 8;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
    float* stage = reinterpret_cast<float*>(smem + L::STG_OFF + quarter * L::STAGE_BYTES);
    const bool lane_ok = lane < L::FPW;
    bool ok = true;
    // dropout: keep bits of the tiles ahead, walking this CTA's tiles (they may belong to later items)
    BwdTileCursor ahead;
    if (DROPOUT) {
      ok = ahead.start(p, queue, wc);
      for (int s2 = 0; ok && s2 < 2 && ahead.valid; ++s2) {   // the first two tiles
        keep_smem[s2 * 128 + r] =
            keep_bits_row(p, ahead.it.row_base, (ahead.it.q_first + ahead.t) * 128, ahead.it.k0, r);
        __syncwarp();
        if (lane == 0) mbar_arrive(&keep_full[s2]);
        ok = ahead.advance(p, queue, wc);
      }
    }
    int g = 0, gi = 0;   // query tiles and items with tiles so far (barrier phases)
    for (int n = 0; ok; ++n) {
      int id;
      if (!queue.peek(n, id, wc)) { ok = false; break; }
      queue.release(n, lane);
      if (id < 0) break;
      const BwdItem itm = bwd_item(p, id);
      const int key = itm.k0 + r;
      for (int t = 0; t < itm.n_iter; ++t, ++g) {
        const int qrow0 = (itm.q_first + t) * 128;
        if (!DQ) {   // only the keep bits: wait until the compute warps have read those of tile g.
          // (Not ds_full: the compute warps may complete two more tiles before this warp waits,
          // and a parity wait cannot tell a barrier two phases on from one that has not moved.
          // keep_empty of tile g + 2 needs the bits made here, so it cannot run ahead.)
          if (DROPOUT && ahead.valid) {
            if (!warp_wait(&keep_empty[g & 1], (g >> 1) & 1, wc)) { ok = false; break; }
            keep_smem[(g & 1) * 128 + r] =
                keep_bits_row(p, ahead.it.row_base, (ahead.it.q_first + ahead.t) * 128, ahead.it.k0, r);
            __syncwarp();
            if (lane == 0) mbar_arrive(&keep_full[g & 1]);
            if (!ahead.advance(p, queue, wc)) { ok = false; break; }
          }
          continue;
        }
        if (!warp_wait(dq_full, g & 1, wc)) { ok = false; break; }
        tc_fence_after();
        uint32_t gq[128];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          tmem_ld32(lane_base + L::DQT_COL + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&gq[32 * c]));
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < 4; ++h) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&gq[h * 32]));
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(dq_empty);
#pragma unroll
        for (int rd = 0; rd < L::ROUNDS; ++rd) {
          // the previous reduction from this staging slice must have read it
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
          if (lane_ok) {
#pragma unroll
            for (int c = 0; c < L::QPR; ++c) stage[c * L::FPW + lane] = __uint_as_float(gq[rd * L::QPR + c]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {   // rows past N are outside the tensor map and are not written
            tma_reduce_add_3d(&tm_dq, stage, quarter * L::FPW, qrow0 + rd * L::QPR, itm.bh);
            bulk_commit();
          }
        }
        // the compute warps have finished tile g (dq_full follows ds_full): its keep-bit stage is
        // free for the tile two ahead
        if (DROPOUT && ahead.valid) {
          keep_smem[(g & 1) * 128 + r] =
              keep_bits_row(p, ahead.it.row_base, (ahead.it.q_first + ahead.t) * 128, ahead.it.k0, r);
          __syncwarp();
          if (lane == 0) mbar_arrive(&keep_full[g & 1]);
          if (!ahead.advance(p, queue, wc)) { ok = false; break; }
        }
      }
      if (!ok) break;
      // ---- dK epilogue
      if (!warp_wait(fin, gi & 1, wc)) { ok = false; break; }
      ++gi;
      tc_fence_after();
      const float s = p.scale;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t kr[32];
        tmem_ld32(lane_base + L::DK_COL + c * 32, kr);
        tmem_ld_wait();
        reg_fence32(kr);
        if (key < p.N) store_row32(p.dk + (itm.row_base + key) * D + c * 32, kr, s, p.out_align32);
      }
      // the accumulator has been read: the next item's first dK may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dk_free);
    }
    if (lane == 0) bulk_wait0();   // every reduction has completed before the kernel ends
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 13) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace fa
