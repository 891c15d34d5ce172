// Exact attention forward for sm_100a: TMA-staged bf16 tiles, tcgen05 MMAs accumulating in
// TMEM, online softmax with a running row max m and row sum l ("48 FlashAttention", block
// "Tiling и online softmax": m <- max(m, m_block), l and O re-expressed against the new m), so
// the N x N score matrix never reaches HBM.
//
// One CTA computes one work item (b, h, 128-row query tile) and loops over 128-key blocks.
//   warps 0-3  softmax: thread r owns query row r (= TMEM lane r); masks, exponentiates,
//              writes P (bf16) to TMEM, rescales O when needed, writes O and lse at the end
//   warp 4     producer: TMA loads of the Q tile and the K/V ring (STAGES deep)
//   warp 5     MMA issuer: S = Q K^T into one of two TMEM score buffers, O += P V
// TMEM columns: S0 [0,128) S1 [128,256) O [256,256+D) P0, P1 (64 columns of packed bf16 each).
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
  int causal;
  float scale_log2;            // tau * log2(e)
  int dropout;                 // 0 / 1
  uint32_t drop_thr;
  float drop_scale;            // 1 / (1 - p)
  uint64_t seed;
  uint64_t wait_ns;
  int debug_flags;             // bit 0: producer skips the first K/V load (exercises the timeout path)
};

constexpr float kRescaleThreshold = 8.0f;   // log2 domain
constexpr float kLn2 = 0.69314718055994530942f;

template <int D>
struct FwdLayout {
  static constexpr int TILE = 128 * D * 2;    // bytes of one 128-row bf16 tile (Q, K or V)
  static constexpr int SUB = 128 * 128;       // one 64-column (128-byte) swizzle panel of a tile
  static constexpr int STAGES = (D == 128) ? 3 : 4;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE;
  static constexpr int V_OFF = K_OFF + STAGES * TILE;
  static constexpr int BAR_OFF = V_OFF + STAGES * TILE;
  static constexpr int NBARS = 1 + 3 * STAGES + 2 + 2 + 2 + 1 + 1;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int S_COL0 = 0, S_COL1 = 128, O_COL = 256, P_COL0 = 256 + D, P_COL1 = 256 + D + 64;
  static constexpr int TMEM_COLS = 512;
  static_assert(P_COL1 + 64 <= TMEM_COLS, "TMEM budget");
  static_assert(BYTES <= 232448, "shared memory budget");
};

template <int D, bool DROPOUT>
__global__ void __launch_bounds__(192, 1)
fa_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using L = FwdLayout<D>;
  constexpr int STAGES = L::STAGES;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((smem_u32(smem) & 1023u) != 0) {   // 128-byte swizzle atoms need 1024-byte alignment
    if (tid == 0) record_status(kStatusBadSmemAlign);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;
  uint64_t* v_full = k_full + STAGES;
  uint64_t* kv_empty = v_full + STAGES;
  uint64_t* s_full = kv_empty + STAGES;
  uint64_t* s_empty = s_full + 2;
  uint64_t* p_full = s_empty + 2;
  uint64_t* o_done = p_full + 2;
  uint64_t* fin = o_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

  // ---- work item: longest causal rows first
  const int qt = p.n_qtiles - 1 - int(blockIdx.x);
  const int bh = blockIdx.y;
  const int b = bh / p.H;
  const int q0 = qt * 128;
  int kv_end = p.N;
  if (p.key_lens != nullptr) kv_end = min(kv_end, max(p.key_lens[b], 0));
  if (p.causal) kv_end = min(kv_end, q0 + 128);
  const int n_kv = (kv_end + 127) / 128;

  if (tid == 0) {
    mbar_init(q_full, 1);
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&k_full[s], 1);
      mbar_init(&v_full[s], 1);
      mbar_init(&kv_empty[s], 1);
    }
    for (int s = 0; s < 2; ++s) {
      mbar_init(&s_full[s], 1);
      mbar_init(&s_empty[s], 4);
      mbar_init(&p_full[s], 4);
    }
    mbar_init(o_done, 1);
    mbar_init(fin, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, L::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const WaitCtl wc{p.wait_ns, abort_flag};

  if (warp == 4) {
    // =========================================================== producer
    if (lane == 0 && n_kv > 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      mbar_arrive_expect_tx(q_full, L::TILE);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) tma_load_3d(smem + L::Q_OFF + c * L::SUB, &tm_q, q_full, c * 64, q0, bh);
      int issued = 0;
      for (int j = 0; j < n_kv; ++j) {
        const int st = j % STAGES;
        if (j >= STAGES && !mbar_wait(&kv_empty[st], ((j / STAGES) - 1) & 1, wc)) break;
        if ((p.debug_flags & 1) && j == 0) break;   // test hook: never deliver block 0
        mbar_arrive_expect_tx(&k_full[st], L::TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::K_OFF + st * L::TILE + c * L::SUB, &tm_k, &k_full[st], c * 64, j * 128, bh);
        mbar_arrive_expect_tx(&v_full[st], L::TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::V_OFF + st * L::TILE + c * L::SUB, &tm_v, &v_full[st], c * 64, j * 128, bh);
        issued = j + 1;
      }
      // every copy this thread started must land before the CTA releases its shared memory
      mbar_drain(q_full, 0, p.wait_ns);
      for (int j = max(0, issued - STAGES); j < issued; ++j) {
        mbar_drain(&k_full[j % STAGES], (j / STAGES) & 1, p.wait_ns);
        mbar_drain(&v_full[j % STAGES], (j / STAGES) & 1, p.wait_ns);
      }
    }
    __syncwarp();
  } else if (warp == 5) {
    // =========================================================== MMA issuer
    if (lane == 0 && n_kv > 0) {
      constexpr uint32_t kIdS = idesc_bf16(128, 128, false, false);   // Q: K-major, K: K-major
      constexpr uint32_t kIdPV = idesc_bf16(128, D, false, true);     // P: TMEM, V: MN-major
      const uint32_t q_base = smem_u32(smem + L::Q_OFF);
      auto issue_pv = [&](int t) -> bool {
        const int st = t % STAGES, sb = t & 1;
        if (!mbar_wait(&p_full[sb], (t >> 1) & 1, wc)) return false;
        if (!mbar_wait(&v_full[st], (t / STAGES) & 1, wc)) return false;
        tc_fence_after();
        const uint32_t v_base = smem_u32(smem + L::V_OFF + st * L::TILE);
        const uint32_t p_col = sb ? L::P_COL1 : L::P_COL0;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // 16 keys per step: 8 packed TMEM columns, 2 swizzle atoms of V
          mma_ts(tmem + L::O_COL, tmem + p_col + kk * 8, sdesc_sw128(v_base + kk * 2048, L::SUB, 1024), kIdPV,
                 (t > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&kv_empty[st]);
        mma_commit(o_done);
        return true;
      };
      bool ok = mbar_wait(q_full, 0, wc);
      for (int j = 0; ok && j < n_kv; ++j) {
        const int st = j % STAGES, sb = j & 1;
        if (!mbar_wait(&k_full[st], (j / STAGES) & 1, wc)) { ok = false; break; }
        if (j >= 2 && !mbar_wait(&s_empty[sb], ((j - 2) >> 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
        const uint32_t k_base = smem_u32(smem + L::K_OFF + st * L::TILE);
        const uint32_t s_col = sb ? L::S_COL1 : L::S_COL0;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {   // 16 features per step: 32 bytes inside a 128-byte row
          const uint32_t off = (kk >> 2) * L::SUB + (kk & 3) * 32;
          mma_ss(tmem + s_col, sdesc_sw128(q_base + off, 16, 1024), sdesc_sw128(k_base + off, 16, 1024), kIdS,
                 kk > 0 ? 1u : 0u);
        }
        mma_commit(&s_full[sb]);
        if (j >= 1 && !issue_pv(j - 1)) { ok = false; break; }
      }
      if (ok) issue_pv(n_kv - 1);
      mma_commit(fin);   // completes when every MMA issued above has finished
      mbar_drain(fin, 0, p.wait_ns);
    }
    __syncwarp();
  } else {
    // =========================================================== softmax / epilogue (warps 0-3)
    const int r = tid;
    const int q_row = q0 + r;
    const uint32_t lane_base = tmem + (uint32_t(warp * 32) << 16);
    const float sl2 = p.scale_log2;
    const uint64_t drop_row = (uint64_t(bh) * uint64_t(p.N) + uint64_t(q_row)) * uint64_t(p.N);
    float m_ref = -INFINITY;   // reference max, exp2 domain
    float l = 0.f;
    bool ok = true;
    for (int j = 0; j < n_kv; ++j) {
      const int sb = j & 1;
      if (!mbar_wait(&s_full[sb], (j >> 1) & 1, wc)) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[128];
      {
        const uint32_t s_addr = lane_base + (sb ? L::S_COL1 : L::S_COL0);
        tmem_ld32(s_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        tmem_ld32(s_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        tmem_ld32(s_addr + 64, *reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        tmem_ld32(s_addr + 96, *reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
        tmem_ld_wait();
        reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
        reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
        reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[64]));
        reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[96]));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_empty[sb]);

      const int k0 = j * 128;
      if ((k0 + 128 > kv_end) || (p.causal && k0 + 128 > q0)) {   // block straddles a mask edge
        const int lim = min(kv_end, p.causal ? q_row + 1 : kv_end) - k0;   // columns < lim are kept
#pragma unroll
        for (int c = 0; c < 128; ++c)
          if (c >= lim) sr[c] = __float_as_uint(-INFINITY);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 128; ++c) mx = fmaxf(mx, __uint_as_float(sr[c]));
      const float m_cand = mx * sl2;
      float alpha = 1.f;
      if (m_cand > m_ref + kRescaleThreshold) {
        alpha = ex2_approx(m_ref - m_cand);
        m_ref = m_cand;
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      float rs = 0.f;
      uint32_t pk[64];
#pragma unroll
      for (int c = 0; c < 64; ++c) {
        float p0 = ex2_approx(fmaf(__uint_as_float(sr[2 * c]), sl2, -m_use));
        float p1 = ex2_approx(fmaf(__uint_as_float(sr[2 * c + 1]), sl2, -m_use));
        rs += p0 + p1;
        if (DROPOUT) {   // Z only; the 1/(1-p) factor is applied in fp32 in the epilogue
          const uint64_t ctr = drop_row + uint64_t(k0 + 2 * c);
          p0 = dropout_keep(p.seed, ctr, p.drop_thr) ? p0 : 0.f;
          p1 = dropout_keep(p.seed, ctr + 1, p.drop_thr) ? p1 : 0.f;
        }
        pk[c] = pack_bf16x2(p0, p1);
      }
      // PV of the previous block must be complete: it frees this P buffer (used two blocks ago)
      // and makes O final up to block j-1 before it is rescaled.
      if (j >= 1) {
        if (!mbar_wait(o_done, (j - 1) & 1, wc)) { ok = false; break; }
        tc_fence_after();
      }
      {
        const uint32_t p_addr = lane_base + (sb ? L::P_COL1 : L::P_COL0);
        tmem_st32(p_addr + 0, *reinterpret_cast<uint32_t(*)[32]>(&pk[0]));
        tmem_st32(p_addr + 32, *reinterpret_cast<uint32_t(*)[32]>(&pk[32]));
      }
      if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orr[32];
          tmem_ld32(lane_base + L::O_COL + c * 32, orr);
          tmem_ld_wait();
          reg_fence32(orr);
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
          tmem_st32(lane_base + L::O_COL + c * 32, orr);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
      l = l * alpha + rs;
    }

    // ---- epilogue: O / l -> bf16, lse = (m + log2 l) * ln 2
    const bool row_valid = q_row < p.N;
    __nv_bfloat16* orow = p.o + (uint64_t(bh) * uint64_t(p.N) + uint64_t(row_valid ? q_row : 0)) * D;
    if (n_kv == 0) {
      if (row_valid) {
#pragma unroll
        for (int c = 0; c < D / 8; ++c) reinterpret_cast<uint4*>(orow)[c] = make_uint4(0, 0, 0, 0);
        p.lse[uint64_t(bh) * p.N + q_row] = -INFINITY;
      }
    } else if (ok && mbar_wait(o_done, (n_kv - 1) & 1, wc)) {
      tc_fence_after();
      const float inv_l = l > 0.f ? (DROPOUT ? p.drop_scale : 1.f) / l : 0.f;
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t orr[32];
        tmem_ld32(lane_base + L::O_COL + c * 32, orr);
        tmem_ld_wait();
        reg_fence32(orr);
        uint32_t packed[16];
#pragma unroll
        for (int e = 0; e < 16; ++e)
          packed[e] = pack_bf16x2(__uint_as_float(orr[2 * e]) * inv_l, __uint_as_float(orr[2 * e + 1]) * inv_l);
        if (row_valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + c * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            dst[e] = make_uint4(packed[4 * e], packed[4 * e + 1], packed[4 * e + 2], packed[4 * e + 3]);
        }
      }
      if (row_valid) p.lse[uint64_t(bh) * p.N + q_row] = l > 0.f ? (m_ref + lg2_approx(l)) * kLn2 : -INFINITY;
    }
  }

  // ---- teardown: every role has drained its asynchronous work
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

}  // namespace fa
