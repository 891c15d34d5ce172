// Exact attention forward for sm_100a: TMA-staged bf16 tiles, tcgen05 MMAs accumulating in
// TMEM, online softmax with a running row max m and row sum l ("48 FlashAttention", block
// "Tiling и online softmax": m <- max(m, m_block), l and O re-expressed against the new m), so
// the N x N score matrix never reaches HBM.
//
// Work item: two adjacent 128-row query tiles A and B of one (b, h); the item loops over 128-key
// blocks and both tiles share every K/V block.  The grid is persistent (one CTA per SM): each CTA
// takes the items of a heavy-first list in snake order (round r: CTA c takes item r*G + c, or
// r*G + G-1-c on odd rounds), and its pipelines run on from one item into the next: the K/V rings
// continue, each next Q tile loads as soon as the last S of its tile has been issued, and the
// next item's first S overlaps the epilogue of the previous one.  Warp roles (three warpgroups):
//   warps 0-3  softmax of tile A, warps 4-7 softmax of tile B: thread r owns query row r of its
//              tile (= TMEM lane r); masks, exponentiates, writes P (bf16) over the tile's score
//              columns, rescales O when needed, writes O and lse at the end
//   warp 8     producer of the K ring, warp 10 of the V ring, warp 11 of the two Q tiles
//   warp 9     MMA issuer, in the order PV_A(j), S_A(j+1), PV_B(j), S_B(j+1): while one tile's
//              softmax runs, the tensor core works on the other tile.  P is handed over in two
//              halves of 64 keys, so the first half of PV runs while the second half of P is made.
// Softmax arithmetic: the scale-and-shift and the row sum use packed f32x2 operations and the row
// max a tree of three-input maxima. Without dropout a quarter of the exponentials take a
// polynomial on the FMA pipe and the rest the MUFU unit (see kFmaPairsPer8); with dropout all go to
// the MUFU unit.
// TMEM columns: S_A [0,128), S_B [128,256) (P over the first 64 columns of each), O_A [256,256+D),
// O_B [256+D,256+2D).  tcgen05 operations from one thread complete in issue order, so S_X(j+1)
// (which overwrites P_X(j)) runs after PV_X(j), and its completion also means PV_X(j) is done.
//
// The running max is only moved when a block's max exceeds it by more than 2^8 in the exp2
// domain; the final O / l uses the same reference max for both, so the result is the same
// exact quantity (the sum is taken against a slightly stale shift, values stay <= 256).
#pragma once
#include <cuda_bf16.h>
#include "sm100.cuh"
#include "dropout_hash.cuh"

namespace fa {

struct FwdParams {
  __nv_bfloat16* o;            // [B,H,N,D]
  float* lse;                  // [B,H,N]
  const int32_t* key_lens;     // [B] or null
  int B, H, N;
  int n_qtiles;
  int n_pairs;                 // ceil(n_qtiles / 2): work items per head
  int causal;
  float scale_log2;            // tau * log2(e)
  int dropout;                 // 0 / 1
  uint32_t drop_thr;
  float drop_scale;            // 1 / (1 - p)
  uint64_t seed;
  uint64_t wait_ns;
  int debug_flags;             // bit 0: producer skips the first K/V load (exercises the timeout path)
  int o_align32;               // o is 32-byte aligned: the epilogue uses 32-byte stores
};

constexpr float kRescaleThreshold = 8.0f;   // log2 domain
constexpr float kLn2 = 0.69314718055994530942f;

template <int D>
struct FwdLayout {
  static constexpr int TILE = 128 * D * 2;    // bytes of one 128-row bf16 tile (Q, K or V)
  static constexpr int SUB = 128 * 128;       // one 64-column (128-byte) swizzle panel of a tile
  static constexpr int KST = (D == 128) ? 3 : 4;   // K ring depth (K is needed one MMA earlier than V)
  static constexpr int VST = (D == 128) ? 2 : 4;   // V ring depth
  static constexpr int QA_OFF = 0;
  static constexpr int QB_OFF = QA_OFF + TILE;
  static constexpr int K_OFF = QB_OFF + TILE;
  static constexpr int V_OFF = K_OFF + KST * TILE;
  static constexpr int BAR_OFF = V_OFF + VST * TILE;
  // q_full[2], q_empty[2], k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[2],
  // p_full[2][2], o_fin[2], o_free[2], fin
  static constexpr int NBARS = 4 + 2 * KST + 2 * VST + 2 + 4 + 2 + 2 + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  __device__ static constexpr int s_col(int x) { return 128 * x; }         // S_A, S_B
  __device__ static constexpr int o_col(int x) { return 256 + D * x; }     // O_A, O_B
  static constexpr int TMEM_COLS = 512;
  static_assert(256 + 2 * D <= TMEM_COLS, "TMEM budget");
  static_assert(BYTES <= 232448, "shared memory budget");
};

// Exponentials of one pair of scores: p = 2^(s * sl2 - m).
__device__ __forceinline__ uint64_t exp2_pair(uint32_t s0, uint32_t s1, uint64_t sl2x2, uint64_t negm2) {
  const uint64_t x = f2_fma(f2_make(__uint_as_float(s0), __uint_as_float(s1)), sl2x2, negm2);
  float x0, x1;
  f2_split(x, x0, x1);
  return f2_make(ex2_approx(x0), ex2_approx(x1));
}

// The same pair on the FMA pipe, so that part of the exponentials leave the MUFU unit (16 results
// per clock per SM). Range reduction (Cody and Waite): x = n + f with n = floor(x), f in [0, 1);
// 2^f by a cubic with p(0) = 1 whose coefficients were fitted for this kernel (minimax relative
// error over [0, 1): 8.6e-5, below the 2^-9 rounding of the bf16 P); 2^n enters by adding n to the
// exponent field. x is clamped to -127 first: the result is then a subnormal or larger, and the
// row sum flushes subnormals, so a fully masked row still sums to exactly 0.
__device__ __forceinline__ uint64_t exp2_pair_fma(uint32_t s0, uint32_t s1, uint64_t sl2x2, uint64_t negm2) {
  constexpr float kC1 = 0.6951166391372681f, kC2 = 0.22764497995376587f, kC3 = 0.07706724107265472f;
  constexpr float kMagic = 12582912.0f;   // 1.5 * 2^23: adding it leaves floor(x) in the low bits
  const uint64_t x = f2_fma(f2_make(__uint_as_float(s0), __uint_as_float(s1)), sl2x2, negm2);
  float x0, x1;
  f2_split(x, x0, x1);
  const uint64_t xc = f2_make(fmaxf(x0, -127.f), fmaxf(x1, -127.f));
  const uint64_t mg = f2_make(kMagic, kMagic);
  const uint64_t t = f2_add_rm(xc, mg);                 // kMagic + floor(x), exactly
  const uint64_t fr = f2_sub(xc, f2_sub(t, mg));        // x - floor(x), exactly
  uint64_t pp = f2_fma(f2_make(kC3, kC3), fr, f2_make(kC2, kC2));
  pp = f2_fma(pp, fr, f2_make(kC1, kC1));
  pp = f2_fma(pp, fr, f2_make(1.f, 1.f));
  float p0, p1, t0, t1;
  f2_split(pp, p0, p1);
  f2_split(t, t0, t1);
  // the low bits of t hold n (two's complement); n << 23 is the exponent increment
  return f2_make(__uint_as_float(__float_as_uint(p0) + (__float_as_uint(t0) << 23)),
                 __uint_as_float(__float_as_uint(p1) + (__float_as_uint(t1) << 23)));
}
// Test kernel: y[i] = 2^x[i] by exp2_pair_fma (scale 1, shift 0), for checking its error bound.
__global__ void __launch_bounds__(256) fa_exp2_fma_test_kernel(const float* x, float* y, int n) {
  const int i = 2 * (int(blockIdx.x) * 256 + int(threadIdx.x));
  if (i >= n) return;
  const float x1 = i + 1 < n ? x[i + 1] : 0.f;
  float y0, y1;
  f2_split(exp2_pair_fma(__float_as_uint(x[i]), __float_as_uint(x1), f2_make(1.f, 1.f), f2_make(0.f, 0.f)), y0, y1);
  y[i] = y0;
  if (i + 1 < n) y[i + 1] = y1;
}

// Of every 8 consecutive score pairs, this many take exp2_pair_fma, the rest the MUFU. Measured:
// at d=64 without dropout, 2 of 8 made the 64k-token causal forward 8.6 % faster (1 or 3 of 8 less
// so); at d=128 (headline causal 2x16x4096x128) 1, 2 and 3 of 8 gave 126 -> 123, 120 and 122 us;
// with dropout the counter hash already fills the integer and FMA pipes and a share made it slower.
template <int D, bool DROPOUT>
constexpr int kFmaPairsPer8 = DROPOUT ? 0 : 2;

// Register split per warpgroup (launch: 384 threads x 168 = 64512 registers):
// 128 x (200 + 200 + 104) = 64512.  Each role lowers or raises its budget first thing.
constexpr int kFwdThreads = 384;
constexpr int kFwdLaunchRegs = 168;   // the host checks the kernel's register count against this
__device__ __forceinline__ void reg_dealloc() { asm volatile("setmaxnreg.dec.sync.aligned.u32 104;\n" ::: "memory"); }
__device__ __forceinline__ void reg_alloc() { asm volatile("setmaxnreg.inc.sync.aligned.u32 200;\n" ::: "memory"); }

// Item k of the heavy-first list: pair (longest causal pairs first) and head.
__device__ __forceinline__ void fwd_item(int k, int n_pairs, int BH, int& pair, int& bh) {
  pair = n_pairs - 1 - k / BH;
  bh = k % BH;
}
// Item taken by CTA c of G in round r (snake order).
__device__ __forceinline__ int fwd_snake(int r, int c, int G) { return r * G + ((r & 1) ? (G - 1 - c) : c); }

template <int D, bool DROPOUT>
__global__ void __launch_bounds__(kFwdThreads, 1)
fa_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using L = FwdLayout<D>;
  constexpr int KST = L::KST, VST = L::VST;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((smem_u32(smem) & 1023u) != 0) {   // 128-byte swizzle atoms need 1024-byte alignment
    if (tid == 0) record_status(kStatusBadSmemAlign);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* q_full = bars;           // [2]: tile A, tile B
  uint64_t* q_empty = q_full + 2;    // [2]
  uint64_t* k_full = q_empty + 2;
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;
  uint64_t* v_empty = v_full + VST;
  uint64_t* s_full = v_empty + VST;   // [2]: tile A, tile B
  uint64_t* p_full = s_full + 2;      // [2][2]: tile, half of the keys
  uint64_t* o_fin = p_full + 4;       // [2]: all PV of the item done
  uint64_t* o_free = o_fin + 2;       // [2]: the epilogue has read O
  uint64_t* fin = o_free + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

  const int G = int(gridDim.x), cta = int(blockIdx.x);
  const int BH = p.B * p.H;
  const int n_items = p.n_pairs * BH;
  // per item and tile x: first query row, key limit, number of 128-key blocks
  auto kv_lim_of = [&](int bh) {
    int lim = p.N;
    if (p.key_lens != nullptr) lim = min(lim, max(p.key_lens[bh / p.H], 0));
    return lim;
  };
  auto tile_q0 = [&](int pair, int x) { return (2 * pair + x) * 128; };
  auto tile_kv_end = [&](int pair, int bh, int x) {
    const int lim = kv_lim_of(bh);
    return p.causal ? min(lim, tile_q0(pair, x) + 128) : lim;
  };
  auto tile_n_kv = [&](int pair, int bh, int x) {
    return tile_q0(pair, x) < p.N ? (tile_kv_end(pair, bh, x) + 127) / 128 : 0;
  };

  if (tid == 0) {
    for (int x = 0; x < 2; ++x) {
      mbar_init(&q_full[x], 1);
      mbar_init(&q_empty[x], 1);
    }
    for (int s = 0; s < KST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&s_full[x], 1);
      mbar_init(&p_full[2 * x], 4);
      mbar_init(&p_full[2 * x + 1], 4);
      mbar_init(&o_fin[x], 1);
      mbar_init(&o_free[x], 4);
    }
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 9) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{p.wait_ns, abort_flag};

  if (warp == 11) {
    // =========================================================== producer of the Q tiles
    reg_dealloc();
    if (lane == 0) {
      prefetch_tmap(&tm_q);
      int nq[2] = {0, 0};   // Q tiles delivered, per tile
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int k = fwd_snake(r, cta, G);
        if (k >= n_items) break;
        int pair, bh;
        fwd_item(k, p.n_pairs, BH, pair, bh);
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          if (tile_n_kv(pair, bh, x) == 0) continue;
          // tile x of this item, once the previous item's last S of tile x has read the buffer
          if (nq[x] >= 1 && !mbar_wait(&q_empty[x], (nq[x] - 1) & 1, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(&q_full[x], L::TILE);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(smem + (x ? L::QB_OFF : L::QA_OFF) + c * L::SUB, &tm_q, &q_full[x], c * 64,
                        tile_q0(pair, x), bh);
          ++nq[x];
        }
      }
#pragma unroll
      for (int x = 0; x < 2; ++x)   // the last copies land before the CTA exits
        if (nq[x] >= 1) mbar_drain(&q_full[x], (nq[x] - 1) & 1, p.wait_ns);
    }
    __syncwarp();
  } else if (warp == 8 || warp == 10) {
    // =========================================================== producers of the K (warp 8) and V (warp 10) rings
    reg_dealloc();
    const bool is_k = (warp == 8);
    if (lane == 0) {
      const int NS = is_k ? KST : VST;
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      uint8_t* ring = smem + (is_k ? L::K_OFF : L::V_OFF);
      prefetch_tmap(map);
      int g = 0;            // blocks delivered on this ring so far (all items)
      bool ok = true;
      for (int r = 0; ok; ++r) {
        const int k = fwd_snake(r, cta, G);
        if (k >= n_items) break;
        int pair, bh;
        fwd_item(k, p.n_pairs, BH, pair, bh);
        const int n_max = max(tile_n_kv(pair, bh, 0), tile_n_kv(pair, bh, 1));
        for (int j = 0; j < n_max; ++j, ++g) {
          const int st = g % NS;
          if (g >= NS && !mbar_wait(&empty[st], ((g / NS) - 1) & 1, wc)) { ok = false; break; }
          if ((p.debug_flags & 1) && g == 0) { ok = false; break; }   // test hook: never deliver block 0
          mbar_arrive_expect_tx(&full[st], L::TILE);
#pragma unroll
          for (int c = 0; c < D / 64; ++c)
            tma_load_3d(ring + st * L::TILE + c * L::SUB, map, &full[st], c * 64, j * 128, bh);
        }
      }
      // every copy this thread started must land before the CTA releases its shared memory
      for (int j = max(0, g - NS); j < g; ++j) mbar_drain(&full[j % NS], (j / NS) & 1, p.wait_ns);
    }
    __syncwarp();
  } else if (warp == 9) {
    // =========================================================== MMA issuer
    // The whole warp runs the loop (descriptors stay warp-uniform); the lane that elect.sync picks
    // issues every MMA and commit, so one thread owns all tcgen05 work and each commit covers
    // every MMA before it.
    reg_dealloc();
    auto wait = [&](uint64_t* bar, uint32_t parity) { return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc)); };
    constexpr uint32_t kIdS = idesc_bf16(128, 128, false, false);   // Q: K-major, K: K-major
    constexpr uint32_t kIdPV = idesc_bf16(128, D, false, true);     // P: TMEM, V: MN-major
    // descriptors: low word = s0 + (byte offset in shared memory >> 4) + leading-offset field
    const uint32_t s0 = smem_u32(smem) >> 4;
    constexpr uint32_t kHi = sdesc_sw128_hi(1024), kKM = sdesc_lbo(16), kMN = sdesc_lbo(L::SUB);
    int gk = 0, gv = 0;        // K and V blocks consumed (all items)
    int nb[2] = {0, 0};        // blocks of each tile so far: phase of s_full / p_full
    int ni[2] = {0, 0};        // items with work for each tile so far: phase of o_fin / o_free
    int nq[2] = {0, 0};        // Q tiles consumed, per tile
    bool ok = true;
    for (int r = 0; ok; ++r) {
      const int k = fwd_snake(r, cta, G);
      if (k >= n_items) break;
      int pair, bh;
      fwd_item(k, p.n_pairs, BH, pair, bh);
      const int n_a = tile_n_kv(pair, bh, 0), n_b = tile_n_kv(pair, bh, 1);
      const int n_max = max(n_a, n_b);
      if (n_max == 0) continue;
      auto issue_s = [&](int x, int kst) {   // S_x = Q_x K^T, K in ring stage kst
        const uint32_t q_lo = s0 + uint32_t((x ? L::QB_OFF : L::QA_OFF) >> 4) + kKM;
        const uint32_t k_lo = s0 + uint32_t((L::K_OFF + kst * L::TILE) >> 4) + kKM;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {   // 16 features per step: 32 bytes inside a 128-byte row
          const uint32_t off = ((kk >> 2) * L::SUB + (kk & 3) * 32) >> 4;
          mma_ss_elect(tmem + L::s_col(x), sdesc_join(q_lo + off, kHi), sdesc_join(k_lo + off, kHi), kIdS,
                      kk > 0 ? 1u : 0u);
        }
      };
      auto issue_pv_half = [&](int x, int vst, int h, uint32_t acc0) {   // O_x += P_x[keys of half h] V[same keys]
        const uint32_t v_lo = s0 + uint32_t((L::V_OFF + vst * L::TILE) >> 4) + kMN;
#pragma unroll
        for (int kk = 4 * h; kk < 4 * h + 4; ++kk)   // 16 keys per step: 8 packed TMEM columns, 2 atoms of V
          mma_ts_elect(tmem + L::o_col(x), tmem + L::s_col(x) + kk * 8, sdesc_join(v_lo + kk * (2048 >> 4), kHi),
                      kIdPV, kk > 0 ? 1u : acc0);
      };
      if (!wait(&k_full[gk % KST], (gk / KST) & 1)) { ok = false; break; }
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        if ((x ? n_b : n_a) == 0) continue;
        if (!wait(&q_full[x], nq[x] & 1)) { ok = false; break; }
        ++nq[x];
        tc_fence_after();
        issue_s(x, gk % KST);
        mma_commit_elect(&s_full[x]);
        if (1 == (x ? n_b : n_a)) mma_commit_elect(&q_empty[x]);   // the next item's Q_x may load now
      }
      if (!ok) break;
      mma_commit_elect(&k_empty[gk % KST]);
      for (int j = 0; ok && j < n_max; ++j) {
        const int vst = (gv + j) % VST, kst1 = (gk + j + 1) % KST;
        if (!wait(&v_full[vst], ((gv + j) / VST) & 1)) { ok = false; break; }
        bool have_k = false;   // K_{j+1} resident
#pragma unroll
        for (int x = 0; x < 2; ++x) {
          const int n_x = x ? n_b : n_a;
          if (j >= n_x) continue;
          // the first PV of an item overwrites O: the previous item's epilogue must have read it
          if (j == 0 && ni[x] >= 1 && !wait(&o_free[x], (ni[x] - 1) & 1)) { ok = false; break; }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (!wait(&p_full[2 * x + h], (nb[x] + j) & 1)) { ok = false; break; }
            tc_fence_after();
            issue_pv_half(x, vst, h, j > 0 ? 1u : 0u);
          }
          if (!ok) break;
          if (j + 1 < n_x) {
            if (!have_k) {
              if (!wait(&k_full[kst1], ((gk + j + 1) / KST) & 1)) { ok = false; break; }
              tc_fence_after();
              have_k = true;
            }
            issue_s(x, kst1);
            mma_commit_elect(&s_full[x]);
            if (j + 2 == n_x) mma_commit_elect(&q_empty[x]);   // the next item's Q_x may load now
          } else {
            mma_commit_elect(&o_fin[x]);
          }
        }
        if (!ok) break;
        mma_commit_elect(&v_empty[vst]);                       // V_j: both tiles' PV issued
        if (j + 1 < n_max) mma_commit_elect(&k_empty[kst1]);   // K_{j+1}: both tiles' S issued
      }
      gk += n_max;
      gv += n_max;
      nb[0] += n_a;
      nb[1] += n_b;
      ni[0] += (n_a > 0);
      ni[1] += (n_b > 0);
    }
    mma_commit_elect(fin);   // completes when every MMA issued above has finished
    if (lane == 0) mbar_drain(fin, 0, p.wait_ns);
    __syncwarp();
  } else {
    // =========================================================== softmax / epilogue (warps 0-7)
    reg_alloc();
    const int x = warp >> 2;   // tile
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(quarter * 32) << 16);
    const uint32_t s_addr = lane_base + L::s_col(x);
    const uint32_t o_addr = lane_base + L::o_col(x);
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2_make(sl2, sl2);
    int nb = 0, ni = 0;   // blocks and items of this tile so far (barrier phases)
    bool ok = true;
    for (int rr = 0; ok; ++rr) {
      const int k = fwd_snake(rr, cta, G);
      if (k >= n_items) break;
      int pair, bh;
      fwd_item(k, p.n_pairs, BH, pair, bh);
      const int q0x = tile_q0(pair, x);
      const int q_row = q0x + r;
      const int n = tile_n_kv(pair, bh, x);
      const int kv_x = tile_kv_end(pair, bh, x);
      // counter-hash state of the draw of keys 0-3 of this row; keys 4u..4u+3 add u * gamma
      const uint64_t z_row =
          DROPOUT ? dropout_z(p.seed, (uint64_t(bh) * uint64_t(p.N) + uint64_t(q_row)) * dropout_row_draws(p.N)) : 0ull;
      const uint32_t drop_c = dropout_lane_c(p.drop_thr);
      float m_ref = -INFINITY;   // reference max, exp2 domain
      float l = 0.f;
      for (int j = 0; j < n; ++j) {
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[x], (nb + j) & 1, wc))) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[128];
        tmem_ld32(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < 4; ++h) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32 * h]));

        const int k0 = j * 128;
        if ((k0 + 128 > kv_x) || (p.causal && k0 + 128 > q0x)) {   // block straddles a mask edge
          const int lim = min(kv_x, p.causal ? q_row + 1 : kv_x) - k0;   // columns < lim are kept
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
        }
        float mxv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};   // four independent chains
#pragma unroll
        for (int c = 0; c < 128; c += 8)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            mxv[u] = max3f(mxv[u], __uint_as_float(sr[c + 2 * u]), __uint_as_float(sr[c + 2 * u + 1]));
        const float mx = fmaxf(max3f(mxv[0], mxv[1], mxv[2]), mxv[3]);
        const float m_cand = mx * sl2;
        float alpha = 1.f;
        if (m_cand > m_ref + kRescaleThreshold) {
          alpha = ex2_approx(m_ref - m_cand);
          m_ref = m_cand;
        }
        const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
        const uint64_t negm2 = f2_make(-m_use, -m_use);
        uint64_t rs2 = f2_make(0.f, 0.f);
        const uint64_t z_blk = z_row + uint64_t(k0 >> 2) * kDropGamma;
#pragma unroll
        for (int h = 0; h < 2; ++h) {   // two halves of 64 keys; the MMA takes each half as soon as it is ready
          uint32_t pk[32];
          uint32_t dm_hi = 0u;   // dropout: keep mask of keys 4u+2, 4u+3 (the draw's high word)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int c = 32 * h + e;   // pair index: keys 2c, 2c+1
            const uint64_t pp = (e % 8) >= 8 - kFmaPairsPer8<D, DROPOUT>
                                    ? exp2_pair_fma(sr[2 * c], sr[2 * c + 1], sl2x2, negm2)
                                    : exp2_pair(sr[2 * c], sr[2 * c + 1], sl2x2, negm2);
            rs2 = kFmaPairsPer8<D, DROPOUT> > 0 ? f2_add_ftz(rs2, pp) : f2_add(rs2, pp);
            float p0, p1;
            f2_split(pp, p0, p1);
            pk[e] = pack_bf16x2(p0, p1);
            if (DROPOUT) {   // Z only; the 1/(1-p) factor is applied in fp32 in the epilogue
              if ((c & 1) == 0) {   // one draw for keys 2c .. 2c+3
                const uint64_t x = dropout_mix(z_blk + uint64_t(c >> 1) * kDropGamma);
                dm_hi = dropout_mask2(dropout_flags(uint32_t(x >> 32), drop_c));
                pk[e] &= dropout_mask2(dropout_flags(uint32_t(x), drop_c));
              } else {
                pk[e] &= dm_hi;
              }
            }
          }
          // P over the score columns already read; O already holds PV up to block j-1
          tmem_st32(s_addr + 32 * h, pk);
          if (h == 0 && j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
              uint32_t orr[32];
              tmem_ld32(o_addr + c * 32, orr);
              tmem_ld_wait();
              reg_fence32(orr);
#pragma unroll
              for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
              tmem_st32(o_addr + c * 32, orr);
            }
          }
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&p_full[2 * x + h]);
        }
        float rs0, rs1;
        f2_split(rs2, rs0, rs1);
        l = l * alpha + (rs0 + rs1);
      }
      if (!ok) break;

      // ---- epilogue: O / l -> bf16, lse = (m + log2 l) * ln 2
      const bool row_valid = q_row < p.N;
      __nv_bfloat16* orow = p.o + (uint64_t(bh) * uint64_t(p.N) + uint64_t(row_valid ? q_row : 0)) * D;
      if (n == 0) {
        if (row_valid) {
#pragma unroll
          for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(orow)[c] = make_uint4(0, 0, 0, 0);
          p.lse[uint64_t(bh) * p.N + q_row] = -INFINITY;
        }
        continue;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&o_fin[x], ni & 1, wc))) { ok = false; break; }
      tc_fence_after();
      const float inv_l = l > 0.f ? (DROPOUT ? p.drop_scale : 1.f) / l : 0.f;
      uint32_t packed[D / 2];
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t orr[32];
        tmem_ld32(o_addr + c * 32, orr);
        tmem_ld_wait();
        reg_fence32(orr);
#pragma unroll
        for (int e = 0; e < 16; ++e)
          packed[16 * c + e] =
              pack_bf16x2(__uint_as_float(orr[2 * e]) * inv_l, __uint_as_float(orr[2 * e + 1]) * inv_l);
      }
      // O is in registers: the next item's first PV may overwrite it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[x]);
      if (row_valid) {
        if (p.o_align32) {
#pragma unroll
          for (int e = 0; e < D / 16; ++e)
            st_global_v8(orow + 16 * e, packed[8 * e], packed[8 * e + 1], packed[8 * e + 2], packed[8 * e + 3],
                         packed[8 * e + 4], packed[8 * e + 5], packed[8 * e + 6], packed[8 * e + 7]);
        } else {
          uint4* dst = reinterpret_cast<uint4*>(orow);
#pragma unroll
          for (int e = 0; e < D / 8; ++e)
            dst[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
        }
        p.lse[uint64_t(bh) * p.N + q_row] = l > 0.f ? (m_ref + lg2_approx(l)) * kLn2 : -INFINITY;
      }
      nb += n;
      ++ni;
    }
  }

  // ---- teardown: every role has drained its asynchronous work
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace fa
