// dQ in a pass of its own (the "separate pass" the path allows for dQ besides the fused fp32
// accumulation): query-tile-major, so dQ of a tile accumulates in TMEM across its key blocks and is
// written once, in bf16, with no fp32 reductions through L2.  The price is recomputing S and dP per
// (query tile, key block): three matmuls here, plus the four of the dK/dV pass (fa_bwd_sm100_kernel
// without DQ), against five for the fused path.  Each probability block is rebuilt from Q, K and the
// saved logsumexp ("48 FlashAttention", block "Tiling и online softmax", paragraph "Backward — тоже
// без N×N"):
//   P = exp(S - lse) (masked),  dP = dO V^T,  dS = P * (dP Z/(1-p) - D),  dQ = tau dS K.
//
// Work item: one 128-row query tile of one (b, h); persistent grid, heavy-first snake order.
// Warps: 0-3 compute (thread r = query row r, TMEM lane r); 4 producer of Q, dO and the K ring; 5
// producer of the V ring; 6 MMA issuer; 7 idle.
// TMEM: S0 [0,128), S1 [128,256) (dS, bf16, over the first 64 columns of its block's buffer),
// dP [256,384), dQ [384, 384+D).  MMA order per key block j:
//   dP(j+1) as soon as the compute warps have read dP(j); dQ += dS(j) K_j (A from TMEM);
//   S(j+2) into the buffer dQ(j) has just read.
#pragma once
#include <cuda_bf16.h>
#include "bwd_sm100.cuh"   // kLog2e
#include "dropout_hash.cuh"
#include "sm100.cuh"

namespace fa {

template <int D>
struct DqLayout {
  static constexpr int TILE = 128 * D * 2;
  static constexpr int SUB = 128 * 128;
  // K is read by S(j) and dQ(j), and S(j+2) is issued right after dQ(j): a third K stage lets
  // K_{j+2} load one block ahead instead of behind dQ(j)
  static constexpr int KST = 3, VST = 2;
  static constexpr int Q_OFF = 0;
  static constexpr int DO_OFF = Q_OFF + TILE;
  static constexpr int K_OFF = DO_OFF + TILE;
  static constexpr int V_OFF = K_OFF + KST * TILE;
  static constexpr int BAR_OFF = V_OFF + VST * TILE;
  // qd_full, qd_empty, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[2], dp_full,
  // dp_read, ds_full[2], dq_fin, dq_free, fin
  static constexpr int NBARS = 2 + 2 * KST + 2 * VST + 2 + 7;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int DP_COL = 256, DQ_COL = 384;
  static constexpr int TMEM_COLS = 512;
  static_assert(DQ_COL + D <= TMEM_COLS, "TMEM budget");
  static_assert(BYTES <= 232448, "shared memory budget");
};

struct DqParams {
  __nv_bfloat16* dq;           // [B,H,N,D]
  const float* lse;            // [B,H,N]
  const float* dvec;           // [B,H,N]  D = rowsum(dO * O)
  const int32_t* key_lens;     // [B] or null
  int B, H, N;
  int n_qtiles;
  int causal;
  float scale;
  float scale_log2;
  int dropout;
  uint32_t drop_thr;
  float drop_scale;
  uint64_t seed;
  uint64_t wait_ns;
};

template <int D, bool DROPOUT>
__global__ void __launch_bounds__(256, 1)
fa_bwd_dq_pass_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      const DqParams p) {
  using L = DqLayout<D>;
  constexpr int KST = L::KST, VST = L::VST;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((smem_u32(smem) & 1023u) != 0) {
    if (tid == 0) record_status(kStatusBadSmemAlign);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* qd_full = bars;           // Q and dO of the item
  uint64_t* qd_empty = qd_full + 1;
  uint64_t* k_full = qd_empty + 1;
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;
  uint64_t* v_empty = v_full + VST;
  uint64_t* s_full = v_empty + VST;   // [2]: score buffer
  uint64_t* dp_full = s_full + 2;
  uint64_t* dp_read = dp_full + 1;    // the compute warps hold dP(j) in registers
  // [2]: score buffer.  One per buffer, so that the compute warps cannot complete a barrier twice
  // before the MMA warp has waited on it: block j + 2 needs S(j + 2), issued after dQ(j).
  uint64_t* ds_full = dp_read + 1;
  uint64_t* dq_fin = ds_full + 2;     // per item
  uint64_t* dq_free = dq_fin + 1;     // per item
  uint64_t* fin = dq_free + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

  const int G = int(gridDim.x), cta = int(blockIdx.x);
  const int BH = p.B * p.H;
  const int n_items = p.n_qtiles * BH;
  auto item_of = [&](int r, int& qt, int& bh) {   // heavy-first list, snake order
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
  auto n_blk_of = [&](int qt, int bh) { return (kv_end_of(qt, bh) + 127) / 128; };

  if (tid == 0) {
    mbar_init(qd_full, 1);
    mbar_init(qd_empty, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&k_empty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&v_full[s], 1);
      mbar_init(&v_empty[s], 1);
    }
    mbar_init(&s_full[0], 1);
    mbar_init(&s_full[1], 1);
    mbar_init(dp_full, 1);
    mbar_init(dp_read, 4);
    mbar_init(&ds_full[0], 4);
    mbar_init(&ds_full[1], 4);
    mbar_init(dq_fin, 1);
    mbar_init(dq_free, 4);
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
    // =========================================================== producers: Q, dO, K (warp 4); V (warp 5)
    const bool is_k = (warp == 4);
    if (lane == 0) {
      prefetch_tmap(is_k ? &tm_k : &tm_v);
      if (is_k) {
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_do);
      }
      uint64_t* full = is_k ? k_full : v_full;
      uint64_t* empty = is_k ? k_empty : v_empty;
      const CUtensorMap* map = is_k ? &tm_k : &tm_v;
      uint8_t* ring = smem + (is_k ? L::K_OFF : L::V_OFF);
      const int ns = is_k ? KST : VST;
      int g = 0, ni = 0;
      bool ok = true;
      int qt, bh;
      for (int r = 0; ok && item_of(r, qt, bh); ++r) {
        const int n = n_blk_of(qt, bh);
        if (n == 0) continue;
        if (is_k) {   // Q and dO of the item, once the previous item's last MMA has read them
          if (ni >= 1 && !mbar_wait(qd_empty, (ni - 1) & 1, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(qd_full, 2 * L::TILE);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) {
            tma_load_3d(smem + L::Q_OFF + c * L::SUB, &tm_q, qd_full, c * 64, qt * 128, bh);
            tma_load_3d(smem + L::DO_OFF + c * L::SUB, &tm_do, qd_full, c * 64, qt * 128, bh);
          }
        }
        ++ni;
        for (int j = 0; j < n; ++j, ++g) {
          const int st = g % ns;
          if (g >= ns && !mbar_wait(&empty[st], ((g / ns) - 1) & 1, wc)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[st], L::TILE);
#pragma unroll
          for (int c = 0; c < D / 64; ++c) tma_load_3d(ring + st * L::TILE + c * L::SUB, map, &full[st], c * 64, j * 128, bh);
        }
      }
      for (int j = max(0, g - ns); j < g; ++j) mbar_drain(&full[j % ns], (j / ns) & 1, p.wait_ns);
      if (is_k && ni >= 1) mbar_drain(qd_full, (ni - 1) & 1, p.wait_ns);
    }
    __syncwarp();
  } else if (warp == 6) {
    // =========================================================== MMA issuer (whole warp, elect.sync)
    constexpr uint32_t kIdS = idesc_bf16(128, 128, false, false);   // Q (dO) and K (V), K-major
    constexpr uint32_t kIdQ = idesc_bf16(128, D, false, true);      // dS from TMEM, K MN-major
    const uint32_t s0 = smem_u32(smem) >> 4;
    constexpr uint32_t kHi = sdesc_sw128_hi(1024), kKM = sdesc_lbo(16), kMN = sdesc_lbo(L::SUB);
    auto wait = [&](uint64_t* bar, uint32_t parity) { return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc)); };
    auto issue_nt = [&](uint32_t d_col, int a_off, int b_off) {   // D[128 x 128] = A B^T, both K-major
      const uint32_t a_lo = s0 + uint32_t(a_off >> 4) + kKM, b_lo = s0 + uint32_t(b_off >> 4) + kKM;
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t off = ((kk >> 2) * L::SUB + (kk & 3) * 32) >> 4;
        mma_ss_elect(tmem + d_col, sdesc_join(a_lo + off, kHi), sdesc_join(b_lo + off, kHi), kIdS, kk > 0 ? 1u : 0u);
      }
    };
    int gk = 0, gv = 0, gb = 0, ni = 0;
    bool ok = true;
    int qt, bh;
    for (int r = 0; ok && item_of(r, qt, bh); ++r) {
      const int n = n_blk_of(qt, bh);
      if (n == 0) continue;
      if (!wait(qd_full, ni & 1)) { ok = false; break; }
      // S(0), S(1), dP(0)
      for (int j = 0; j < 2 && j < n; ++j) {
        if (!wait(&k_full[(gk + j) % KST], ((gk + j) / KST) & 1)) { ok = false; break; }
        tc_fence_after();
        issue_nt(128 * ((gb + j) & 1), L::Q_OFF, L::K_OFF + ((gk + j) % KST) * L::TILE);
        mma_commit_elect(&s_full[(gb + j) & 1]);
      }
      if (!ok) break;
      // the dP columns: the previous block's dP has been read (it is the previous item's last)
      if (gb >= 1 && !wait(dp_read, (gb - 1) & 1)) { ok = false; break; }
      if (!wait(&v_full[gv % VST], (gv / VST) & 1)) { ok = false; break; }
      tc_fence_after();
      issue_nt(L::DP_COL, L::DO_OFF, L::V_OFF + (gv % VST) * L::TILE);
      mma_commit_elect(dp_full);
      mma_commit_elect(&v_empty[gv % VST]);
      for (int j = 0; ok && j < n; ++j) {
        const int b = gb + j, buf = b & 1;
        // dP(j+1) once the compute warps hold dP(j) in registers
        if (j + 1 < n) {
          if (!wait(dp_read, b & 1)) { ok = false; break; }
          if (!wait(&v_full[(gv + j + 1) % VST], ((gv + j + 1) / VST) & 1)) { ok = false; break; }
          tc_fence_after();
          issue_nt(L::DP_COL, L::DO_OFF, L::V_OFF + ((gv + j + 1) % VST) * L::TILE);
          mma_commit_elect(dp_full);
          mma_commit_elect(&v_empty[(gv + j + 1) % VST]);
        }
        // dQ += dS(j) K_j   (A = dS in TMEM: 16 keys per step = 8 packed columns; B = K_j MN-major)
        if (j == 0 && ni >= 1 && !wait(dq_free, (ni - 1) & 1)) { ok = false; break; }
        if (!wait(&ds_full[buf], (b >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        {
          const uint32_t k_lo = s0 + uint32_t((L::K_OFF + ((gk + j) % KST) * L::TILE) >> 4) + kMN;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts_elect(tmem + L::DQ_COL, tmem + 128 * buf + kk * 8, sdesc_join(k_lo + kk * (2048 >> 4), kHi), kIdQ,
                        (j > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit_elect(&k_empty[(gk + j) % KST]);   // K_j: last read by dQ(j)
        // S(j+2) into the buffer dQ(j) has just read
        if (j + 2 < n) {
          if (!wait(&k_full[(gk + j + 2) % KST], ((gk + j + 2) / KST) & 1)) { ok = false; break; }
          tc_fence_after();
          issue_nt(128 * buf, L::Q_OFF, L::K_OFF + ((gk + j + 2) % KST) * L::TILE);
          mma_commit_elect(&s_full[buf]);
        }
      }
      if (!ok) break;
      mma_commit_elect(dq_fin);
      mma_commit_elect(qd_empty);   // Q and dO: every MMA of the item has read them
      gk += n;
      gv += n;
      gb += n;
      ++ni;
    }
    mma_commit_elect(fin);
    if (lane == 0) mbar_drain(fin, 0, p.wait_ns);
    __syncwarp();
  } else if (warp < 4) {
    // =========================================================== compute (query row r)
    const int r = warp * 32 + lane;
    const uint32_t lane_base = tmem + (uint32_t(warp * 32) << 16);
    const uint64_t sl2x2 = f2_make(p.scale_log2, p.scale_log2);
    int gb = 0, ni = 0;
    bool ok = true;
    int qt, bh;
    for (int rr = 0; ok && item_of(rr, qt, bh); ++rr) {
      const int n = n_blk_of(qt, bh);
      const int q0 = qt * 128, q_row = q0 + r;
      const bool row_valid = q_row < p.N;
      const uint64_t row_base = uint64_t(bh) * uint64_t(p.N);
      const int kv_x = kv_end_of(qt, bh);
      const float nl2 = row_valid ? -p.lse[row_base + q_row] * kLog2e : 0.f;   // -lse, exp2 domain
      const float nd = row_valid ? -p.dvec[row_base + q_row] : 0.f;            // -D
      const uint64_t nl2x2 = f2_make(nl2, nl2), ndx2 = f2_make(nd, nd);
      const uint64_t z_row = DROPOUT ? dropout_z(p.seed, (row_base + uint64_t(q_row)) * dropout_row_draws(p.N)) : 0ull;
      const uint32_t drop_c = dropout_lane_c(p.drop_thr);
      for (int j = 0; j < n; ++j) {
        const int b = gb + j, buf = b & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&s_full[buf], (b >> 1) & 1, wc))) { ok = false; break; }
        tc_fence_after();
        float pr[128];
        {
          uint32_t* sr = reinterpret_cast<uint32_t*>(pr);
#pragma unroll
          for (int c = 0; c < 4; ++c)
            tmem_ld32(lane_base + 128 * buf + 32 * c, *reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
          tmem_ld_wait();
#pragma unroll
          for (int c = 0; c < 4; ++c) reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32 * c]));
        }
        // P = exp2(S tau log2e - lse2), masked
#pragma unroll
        for (int c = 0; c < 128; c += 2) {
          float x0, x1;
          f2_split(f2_fma(f2_make(pr[c], pr[c + 1]), sl2x2, nl2x2), x0, x1);
          pr[c] = ex2_approx(x0);
          pr[c + 1] = ex2_approx(x1);
        }
        const int k0 = 128 * j;
        if ((k0 + 128 > kv_x) || (p.causal && k0 + 128 > q0) || !row_valid) {
          const int lim = row_valid ? min(kv_x, p.causal ? q_row + 1 : kv_x) - k0 : 0;
#pragma unroll
          for (int c = 0; c < 128; ++c)
            if (c >= lim) pr[c] = 0.f;
        }
        if (!__all_sync(0xffffffffu, mbar_wait(dp_full, b & 1, wc))) { ok = false; break; }
        tc_fence_after();
        const uint64_t z_blk = z_row + uint64_t(k0 >> 2) * kDropGamma;
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {   // dS = P (dP Z/(1-p) - D), 64 keys at a time
          uint32_t dr[64];
          tmem_ld32(lane_base + L::DP_COL + 64 * hh, *reinterpret_cast<uint32_t(*)[32]>(&dr[0]));
          tmem_ld32(lane_base + L::DP_COL + 64 * hh + 32, *reinterpret_cast<uint32_t(*)[32]>(&dr[32]));
          tmem_ld_wait();
          reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&dr[0]));
          reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&dr[32]));
          if (hh == 1) {   // dP(j) is in registers: dP(j+1) may overwrite the columns
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dp_read);
          }
          uint32_t pk[32];
          uint32_t fl_hi = 0u;   // dropout: keep flags of keys 4u+2, 4u+3 (the draw's high word)
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int c = 64 * hh + 2 * e;
            float dpa = __uint_as_float(dr[2 * e]), dpb = __uint_as_float(dr[2 * e + 1]);
            if (DROPOUT) {
              uint32_t fl;
              if ((e & 1) == 0) {   // one draw for keys c .. c+3
                const uint64_t x = dropout_mix(z_blk + uint64_t(c >> 2) * kDropGamma);
                fl = dropout_flags(uint32_t(x), drop_c);
                fl_hi = dropout_flags(uint32_t(x >> 32), drop_c);
              } else {
                fl = fl_hi;
              }
              dpa = (fl & 0x8000u) ? dpa * p.drop_scale : 0.f;
              dpb = (fl & 0x80000000u) ? dpb * p.drop_scale : 0.f;
            }
            float da, db;
            f2_split(f2_mul(f2_make(pr[c], pr[c + 1]), f2_add(f2_make(dpa, dpb), ndx2)), da, db);
            pk[e] = pack_bf16x2(da, db);
          }
          // dS over the first 64 score columns of its buffer (scores already read)
          tmem_st32(lane_base + 128 * buf + 32 * hh, pk);
        }
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&ds_full[buf]);
      }
      if (!ok) break;
      // ---- epilogue: dq = bf16(tau * dQ)
      __nv_bfloat16* qrow = p.dq + (row_base + uint64_t(row_valid ? q_row : 0)) * D;
      if (n == 0) {
        if (row_valid) {
#pragma unroll
          for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(qrow)[c] = make_uint4(0, 0, 0, 0);
        }
        continue;
      }
      if (!__all_sync(0xffffffffu, mbar_wait(dq_fin, ni & 1, wc))) { ok = false; break; }
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t orr[32];
        tmem_ld32(lane_base + L::DQ_COL + 32 * c, orr);
        tmem_ld_wait();
        reg_fence32(orr);
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          w[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * p.scale, __uint_as_float(orr[2 * e + 1]) * p.scale);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(qrow + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(w[4 * e], w[4 * e + 1], w[4 * e + 2], w[4 * e + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dq_free);
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
