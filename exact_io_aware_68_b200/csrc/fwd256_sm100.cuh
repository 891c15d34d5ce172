// Exact attention forward for head dimension 256 on sm_100a: the same online softmax as the
// d <= 128 kernel ("48 FlashAttention", block "Tiling и online softmax"), laid out for the larger
// head.  O alone takes 256 of the 512 TMEM columns, so a CTA holds ONE 128-row query tile; to keep
// the tensor core busy while that tile's softmax runs, the scores of the next key block are computed
// into a second TMEM buffer.  Key blocks are 64 keys (a K or V block is 32 KB, so both rings can be
// double-buffered beside the 64 KB Q tile).
//
// Work item: one 128-row query tile of one (b, h); the grid is persistent (one CTA per SM, items in
// heavy-first snake order as in the d <= 128 kernel).  Warps:
//   warps 0-3  softmax: thread r owns query row r (TMEM lane r); per block of 64 keys it masks,
//              takes the row max, moves the reference max (rescaling O, after the P.V in flight has
//              completed) when a block exceeds it by more than 2^8, writes P (bf16) over the first 32
//              columns of the block's score buffer, and at the end writes O / l and lse
//   warp 4     producer of the Q tile and the K ring; warp 5 producer of the V ring
//   warp 6     MMA issuer: S(j) = Q K_j^T (M = 128, N = 64, K = 256) into score buffer j % 2;
//              O += P(j) V_j (M = 128, N = 256, K = 64, P from TMEM); S(j + 2) after P(j) V_j
//   warp 7     idle
// TMEM: S0 [0, 64), S1 [64, 128), O [256, 512).
#pragma once
#include <cuda_bf16.h>
#include "sm100.cuh"
#include "dropout_hash.cuh"

namespace fa {

struct Fwd256Layout {
  static constexpr int D = 256;
  static constexpr int QSUB = 128 * 128;       // one 64-feature panel of the 128-row Q tile
  static constexpr int KSUB = 64 * 128;        // one 64-feature panel of a 64-key K or V block
  static constexpr int QTILE = 4 * QSUB;       // 64 KB
  static constexpr int BLK = 4 * KSUB;         // 32 KB
  static constexpr int KST = 2, VST = 2;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + QTILE;
  static constexpr int V_OFF = K_OFF + KST * BLK;
  static constexpr int BAR_OFF = V_OFF + VST * BLK;
  // q_full, q_empty, k_full[2], k_empty[2], v_full[2], v_empty[2], s_full[2], p_full[2], pv_done,
  // o_fin, o_free, fin
  static constexpr int NBARS = 2 + 2 * KST + 2 * VST + 2 + 2 + 4;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int O_COL = 256;
  static constexpr int TMEM_COLS = 512;
  static_assert(BYTES <= 232448, "shared memory budget");
};

struct Fwd256Params {
  __nv_bfloat16* o;            // [B,H,N,256]
  float* lse;                  // [B,H,N]
  const int32_t* key_lens;     // [B] or null
  int B, H, N;
  int n_qtiles;
  int causal;
  float scale_log2;
  int dropout;
  uint32_t drop_thr;
  float drop_scale;
  uint64_t seed;
  uint64_t wait_ns;
};

constexpr float kRescale256 = 8.0f;   // log2 domain
constexpr float kLn2_256 = 0.69314718055994530942f;

template <bool DROPOUT>
__global__ void __launch_bounds__(256, 1)
fa_fwd256_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const Fwd256Params p) {
  using L = Fwd256Layout;
  constexpr int KST = L::KST, VST = L::VST;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((smem_u32(smem) & 1023u) != 0) {
    if (tid == 0) record_status(kStatusBadSmemAlign);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* q_empty = q_full + 1;
  uint64_t* k_full = q_empty + 1;
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;
  uint64_t* v_empty = v_full + VST;
  uint64_t* s_full = v_empty + VST;   // [2]: score buffer
  uint64_t* p_full = s_full + 2;      // [2]: score buffer
  uint64_t* pv_done = p_full + 2;     // one phase per block
  uint64_t* o_fin = pv_done + 1;      // one phase per item
  uint64_t* o_free = o_fin + 1;       // one phase per item
  uint64_t* fin = o_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

  const int G = int(gridDim.x), cta = int(blockIdx.x);
  const int BH = p.B * p.H;
  const int n_items = p.n_qtiles * BH;
  // item k of the heavy-first list (the longest causal tiles first), taken in snake order
  auto item_of = [&](int r, int& qt, int& bh) {
    const int k = r * G + ((r & 1) ? (G - 1 - cta) : cta);
    qt = p.n_qtiles - 1 - k / BH;
    bh = k % BH;
    return k < n_items;
  };
  auto kv_end_of = [&](int qt, int bh) {
    int lim = p.N;
    if (p.key_lens != nullptr) lim = min(lim, max(p.key_lens[bh / p.H], 0));
    return p.causal ? min(lim, qt * 128 + 128) : lim;
  };
  auto n_blk_of = [&](int qt, int bh) { return (kv_end_of(qt, bh) + 63) / 64; };

  if (tid == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&p_full[s], 4);
    }
    mbar_init(pv_done, 1);
    mbar_init(o_fin, 1);
    mbar_init(o_free, 4);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 6) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{p.wait_ns, abort_flag};

  if (warp == 4 || warp == 5) {
    // =========================================================== producers: Q and K (warp 4), V (warp 5)
    const bool is_k = (warp == 4);
    if (lane == 0) {
      prefetch_tmap(is_k ? &tm_k : &tm_v);
      if (is_k) prefetch_tmap(&tm_q);
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      uint8_t* ring = smem + (is_k ? L::K_OFF : L::V_OFF);
      int g = 0, nq = 0;   // blocks delivered on this ring; Q tiles delivered
      bool ok = true;
      int qt, bh;
      for (int r = 0; ok && item_of(r, qt, bh); ++r) {
        const int n = n_blk_of(qt, bh);
        if (n == 0) continue;
        if (is_k) {   // the Q tile, once the previous item's last S has read the buffer
          if (nq >= 1 && !mbar_wait(q_empty, (nq - 1) & 1, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(q_full, L::QTILE);
#pragma unroll
          for (int c = 0; c < 4; ++c) tma_load_3d(smem + L::Q_OFF + c * L::QSUB, &tm_q, q_full, c * 64, qt * 128, bh);
          ++nq;
        }
        for (int j = 0; j < n; ++j, ++g) {
          const int st = g % (is_k ? KST : VST);
          const int ns = is_k ? KST : VST;
          if (g >= ns && !mbar_wait(&empty[st], ((g / ns) - 1) & 1, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[st], L::BLK);
#pragma unroll
          for (int c = 0; c < 4; ++c) tma_load_3d(ring + st * L::BLK + c * L::KSUB, map, &full[st], c * 64, j * 64, bh);
        }
      }
      // every copy this thread started lands before the CTA releases its shared memory
      const int ns = is_k ? KST : VST;
      for (int j = max(0, g - ns); j < g; ++j) mbar_drain(&full[j % ns], (j / ns) & 1, p.wait_ns);
      if (is_k && nq >= 1) mbar_drain(q_full, (nq - 1) & 1, p.wait_ns);
    }
    __syncwarp();
  } else if (warp == 6) {
    // =========================================================== MMA issuer (whole warp, elect.sync)
    constexpr uint32_t kIdS = idesc_bf16(128, 64, false, false);    // Q, K both K-major
    constexpr uint32_t kIdPV = idesc_bf16(128, 256, false, true);   // P from TMEM, V MN-major
    const uint32_t s0 = smem_u32(smem) >> 4;
    constexpr uint32_t kHi = sdesc_sw128_hi(1024), kKM = sdesc_lbo(16), kMN = sdesc_lbo(L::KSUB);
    auto wait = [&](uint64_t* bar, uint32_t parity) { return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc)); };
    int gk = 0, gv = 0, gb = 0, ni = 0;   // K blocks, V blocks, blocks (all items), items with work
    bool ok = true;
    int qt, bh;
    auto issue_s = [&](int buf, int kst) {   // S = Q K^T into score buffer buf
      const uint32_t q_lo = s0 + uint32_t(L::Q_OFF >> 4) + kKM;
      const uint32_t k_lo = s0 + uint32_t((L::K_OFF + kst * L::BLK) >> 4) + kKM;
#pragma unroll
      for (int kk = 0; kk < 16; ++kk) {   // 16 features per step
        const uint32_t qo = ((kk >> 2) * L::QSUB + (kk & 3) * 32) >> 4;
        const uint32_t ko = ((kk >> 2) * L::KSUB + (kk & 3) * 32) >> 4;
        mma_ss_elect(tmem + 64 * buf, sdesc_join(q_lo + qo, kHi), sdesc_join(k_lo + ko, kHi), kIdS, kk > 0 ? 1u : 0u);
      }
    };
    for (int r = 0; ok && item_of(r, qt, bh); ++r) {
      const int n = n_blk_of(qt, bh);
      if (n == 0) continue;
      if (!wait(q_full, ni & 1)) { ok = false; break; }
      // the first two score blocks of the item
      for (int j = 0; j < 2 && j < n; ++j) {
        if (!wait(&k_full[(gk + j) % KST], ((gk + j) / KST) & 1)) { ok = false; break; }
        tc_fence_after();
        issue_s((gb + j) & 1, (gk + j) % KST);
        mma_commit_elect(&s_full[(gb + j) & 1]);
        mma_commit_elect(&k_empty[(gk + j) % KST]);
        if (j + 1 == n) mma_commit_elect(q_empty);
      }
      if (!ok) break;
      for (int j = 0; ok && j < n; ++j) {
        const int b = gb + j, buf = b & 1;
        // O += P(j) V_j; the item's first P.V overwrites O: the previous epilogue must have read it
        if (j == 0 && ni >= 1 && !wait(o_free, (ni - 1) & 1)) { ok = false; break; }
        if (!wait(&p_full[buf], (b >> 1) & 1)) { ok = false; break; }
        if (!wait(&v_full[(gv + j) % VST], ((gv + j) / VST) & 1)) { ok = false; break; }
        tc_fence_after();
        {
          const uint32_t v_lo = s0 + uint32_t((L::V_OFF + ((gv + j) % VST) * L::BLK) >> 4) + kMN;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)   // 16 keys per step: 8 packed TMEM columns
            mma_ts_elect(tmem + L::O_COL, tmem + 64 * buf + kk * 8, sdesc_join(v_lo + kk * (2048 >> 4), kHi),
                        kIdPV, (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit_elect(&v_empty[(gv + j) % VST]);
        mma_commit_elect(pv_done);
        // S(j + 2) into the buffer P(j) V_j has just read (MMAs run in issue order)
        if (j + 2 < n) {
          if (!wait(&k_full[(gk + j + 2) % KST], ((gk + j + 2) / KST) & 1)) { ok = false; break; }
          tc_fence_after();
          issue_s(buf, (gk + j + 2) % KST);
          mma_commit_elect(&s_full[buf]);
          mma_commit_elect(&k_empty[(gk + j + 2) % KST]);
          if (j + 3 == n) mma_commit_elect(q_empty);
        }
      }
      if (!ok) break;
      mma_commit_elect(o_fin);
      gk += n;
      gv += n;
      gb += n;
      ++ni;
    }
    mma_commit_elect(fin);
    if (lane == 0) mbar_drain(fin, 0, p.wait_ns);
    __syncwarp();
  } else if (warp < 4) {
    // =========================================================== softmax / epilogue (warps 0-3)
    const int r = warp * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(warp * 32) << 16);
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2_make(sl2, sl2);
    int gb = 0, ni = 0;
    bool ok = true;
    int qt, bh;
    for (int rr = 0; ok && item_of(rr, qt, bh); ++rr) {
      const int n = n_blk_of(qt, bh);
      const int q0 = qt * 128, q_row = q0 + r;
      const int kv_x = kv_end_of(qt, bh);
      const uint64_t z_row =
          DROPOUT ? dropout_z(p.seed, (uint64_t(bh) * uint64_t(p.N) + uint64_t(q_row)) * dropout_row_draws(p.N)) : 0ull;
      const uint32_t drop_c = dropout_lane_c(p.drop_thr);
      float m_ref = -INFINITY, l = 0.f;
      for (int j = 0; j < n; ++j) {
        const int b = gb + j, buf = b & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[buf], (b >> 1) & 1, wc))) { ok = false; break; }
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(lane_base + 64 * buf, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(lane_base + 64 * buf + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld_wait();
        reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        const int k0 = 64 * j;
        if ((k0 + 64 > kv_x) || (p.causal && k0 + 64 > q0)) {   // the block straddles a mask edge
          const int lim = min(kv_x, p.causal ? q_row + 1 : kv_x) - k0;
#pragma unroll
          for (int c = 0; c < 64; ++c)
            if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
        }
        float mxv[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
        for (int c = 0; c < 64; c += 8)
#pragma unroll
          for (int u = 0; u < 4; ++u)
            mxv[u] = max3f(mxv[u], __uint_as_float(sr[c + 2 * u]), __uint_as_float(sr[c + 2 * u + 1]));
        const float m_cand = fmaxf(max3f(mxv[0], mxv[1], mxv[2]), mxv[3]) * sl2;
        float alpha = 1.f;
        if (m_cand > m_ref + kRescale256) {
          alpha = ex2_approx(m_ref - m_cand);
          m_ref = m_cand;
        }
        // O holds P.V up to block j - 1 once that MMA has completed (it may still be running: the
        // score buffers run two blocks ahead); rescale it, 16 columns at a time
        if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
          if (!__all_sync(0xffffffffu, mbar_wait(pv_done, (b - 1) & 1, wc))) { ok = false; break; }
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 256 / 16; ++c) {
            uint32_t orr[16];
            tmem_ld16(lane_base + L::O_COL + 16 * c, orr);
            tmem_ld_wait();
            reg_fence16(orr);
#pragma unroll
            for (int e = 0; e < 16; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
            tmem_st16(lane_base + L::O_COL + 16 * c, orr);
          }
          tmem_st_wait();
        }
        const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
        const uint64_t negm2 = f2_make(-m_use, -m_use);
        uint64_t rs2 = f2_make(0.f, 0.f);
        const uint64_t z_blk = z_row + uint64_t(k0 >> 2) * kDropGamma;
        uint32_t pk[32];
        uint32_t dm_hi = 0u;   // dropout: keep mask of keys 4u+2, 4u+3 (the draw's high word)
#pragma unroll
        for (int e = 0; e < 32; ++e) {   // pair e: keys 2e, 2e + 1 of the block
          const uint64_t x = f2_fma(f2_make(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])), sl2x2, negm2);
          float x0, x1;
          f2_split(x, x0, x1);
          const uint64_t pp = f2_make(ex2_approx(x0), ex2_approx(x1));
          rs2 = f2_add(rs2, pp);
          float p0, p1;
          f2_split(pp, p0, p1);
          pk[e] = pack_bf16x2(p0, p1);
          if (DROPOUT) {   // Z only; the 1/(1-p) factor is applied in fp32 in the epilogue
            if ((e & 1) == 0) {   // one draw for keys 2e .. 2e+3
              const uint64_t xd = dropout_mix(z_blk + uint64_t(e >> 1) * kDropGamma);
              dm_hi = dropout_mask2(dropout_flags(uint32_t(xd >> 32), drop_c));
              pk[e] &= dropout_mask2(dropout_flags(uint32_t(xd), drop_c));
            } else {
              pk[e] &= dm_hi;
            }
          }
        }
        tmem_st32(lane_base + 64 * buf, pk);   // P over the block's score columns, already read
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&p_full[buf]);
        float rs0, rs1;
        f2_split(rs2, rs0, rs1);
        l = l * alpha + (rs0 + rs1);
      }
      if (!ok) break;
      // ---- epilogue: O / l -> bf16, lse = (m + log2 l) * ln 2
      const bool row_valid = q_row < p.N;
      __nv_bfloat16* orow = p.o + (uint64_t(bh) * uint64_t(p.N) + uint64_t(row_valid ? q_row : 0)) * 256;
      if (n == 0) {
        if (row_valid) {
#pragma unroll
          for (int c = 0; c < 32; ++c) reinterpret_cast<uint4*>(orow)[c] = make_uint4(0, 0, 0, 0);
          p.lse[uint64_t(bh) * p.N + q_row] = -INFINITY;
        }
        continue;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(o_fin, ni & 1, wc))) { ok = false; break; }
      tc_fence_after();
      const float inv_l = l > 0.f ? (DROPOUT ? p.drop_scale : 1.f) / l : 0.f;
#pragma unroll 1
      for (int c = 0; c < 8; ++c) {   // 32 features at a time
        uint32_t orr[32];
        tmem_ld32(lane_base + L::O_COL + 32 * c, orr);
        tmem_ld_wait();
        reg_fence32(orr);
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * inv_l, __uint_as_float(orr[2 * e + 1]) * inv_l);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(o_free);
      if (row_valid) p.lse[uint64_t(bh) * p.N + q_row] = l > 0.f ? (m_ref + lg2_approx(l)) * kLn2_256 : -INFINITY;
      gb += n;
      ++ni;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 6) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace fa
