// Decode-shaped exact attention for sm_100a: Nq new query rows (1..64) of each head against a long
// cache of Nkv keys, the use "48 FlashAttention" (block "Связи") names for the kernel under
// vLLM / PagedAttention.  Query i is the token at position L - Nq + i of a cache of L valid keys
// (L = key_lens[b], else Nkv): causal keeps key j <= L - Nq + i, key padding keeps j < L.
//
// The work of one head is a few rows against many keys, so it is split over the key range: CTA
// (s, bh) runs the online softmax of "Tiling и online softmax" (same page) over keys
// [s*C, (s+1)*C) and writes its partial (reference max m, row sum l, unnormalised O) in fp32;
// fa_decode_combine_kernel merges the partials of a head: m* = max m_s, w_s = 2^(m_s - m*),
// O = sum w_s O_s / sum w_s l_s, lse = (m* + log2 sum w_s l_s) ln 2.  Bound: HBM (every K and V byte
// is read once; a row of Nq queries does Nq * 4 d FLOP per key).
//
// Split kernel, 6 warps, an M = 128 tile whose rows r and r + 64 hold the same query row r % 64:
//   warps 0-3  softmax: thread r (TMEM lane r) exponentiates the key half r / 64 of every 128-key
//              block (64 keys) for query row r % 64 and keeps its own running max and sum, so each
//              half of a split's keys is a partial of its own for the combine (2 per CTA); P (bf16:
//              its 64 keys, zeros for the other half) goes over the first 64 columns of the score
//              buffer.  Half the exponentials per thread and block of a one-thread-per-row tile.
//   warp 4     producer: Q twice (tile rows 0-63 and 64-127, zero past Nq), K and V rings
//   warp 5     MMA issuer: S(j) = Q K_j^T (M = 128, N = 128) into one of two TMEM score buffers, so
//              that S(j+1) runs while block j is exponentiated; O += P(j) V_j (M = 128, N = D, P from
//              TMEM)
// TMEM: S0 [0,128), S1 [128,256), O [256, 256+D).
#pragma once
#include <cuda_bf16.h>
#include "sm100.cuh"

namespace fa {

constexpr float kDecodeRescale = 8.0f;   // move the reference max only when a block exceeds it by 2^8
constexpr float kDecodeLn2 = 0.69314718055994530942f;

struct DecodeParams {
  float* part_o;               // [BH][n_part][Nq][D] fp32, unnormalised
  float* part_ml;              // [BH][n_part][Nq][2] fp32: m (log2 domain), l
  __nv_bfloat16* o;            // [B,H,Nq,D]
  float* lse;                  // [B,H,Nq]
  const int32_t* key_lens;     // [B] or null
  int B, H, Nq, Nkv;
  int chunk;                   // keys per split (multiple of 128)
  int n_split;                 // key-range splits per head (CTAs per head)
  int n_part;                  // partials per head: 2 per split (one per key half)
  int causal;
  float scale_log2;
  uint64_t wait_ns;
};

template <int D>
struct DecodeLayout {
  static constexpr int SUB = 128 * 128;          // one 64-column (128-byte) panel of a 128-row tile
  static constexpr int QHALF = 64 * 128;         // rows 64-127 of a panel start here
  static constexpr int TILE = D / 64 * SUB;      // a 128-row bf16 tile (Q, or a K/V block)
  static constexpr int KST = (D == 128) ? 3 : 4;
  static constexpr int VST = (D == 128) ? 2 : 4;
  static constexpr int Q_OFF = 0;
  static constexpr int K_OFF = Q_OFF + TILE;
  static constexpr int V_OFF = K_OFF + KST * TILE;
  static constexpr int BAR_OFF = V_OFF + VST * TILE;
  // q_full, k_full[KST], k_empty[KST], v_full[VST], v_empty[VST], s_full[2], s_free[2], p_full[2],
  // pv_done, fin
  static constexpr int NBARS = 1 + 2 * KST + 2 * VST + 6 + 2;
  static constexpr int MISC_OFF = BAR_OFF + NBARS * 8;
  static constexpr int BYTES = MISC_OFF + 16;
  static constexpr int O_COL = 256;
  static constexpr int TMEM_COLS = 512;
  static_assert(O_COL + D <= TMEM_COLS, "TMEM budget");
  static_assert(BYTES <= 232448, "shared memory budget");
};

template <int D>
__global__ void __launch_bounds__(192, 1)
fa_decode_split_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const DecodeParams p) {
  using L = DecodeLayout<D>;
  constexpr int KST = L::KST, VST = L::VST;
  extern __shared__ __align__(1024) uint8_t smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if ((smem_u32(smem) & 1023u) != 0) {
    if (tid == 0) record_status(kStatusBadSmemAlign);
    return;
  }
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::BAR_OFF);
  uint64_t* q_full = bars;
  uint64_t* k_full = q_full + 1;
  uint64_t* k_empty = k_full + KST;
  uint64_t* v_full = k_empty + KST;
  uint64_t* v_empty = v_full + VST;
  uint64_t* s_full = v_empty + VST;   // [2]
  uint64_t* s_free = s_full + 2;      // [2]: the softmax has read the scores out of the buffer
  uint64_t* p_full = s_free + 2;      // [2]: P is in the buffer
  uint64_t* pv_done = p_full + 2;     // one phase per block
  uint64_t* fin = pv_done + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::MISC_OFF);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::MISC_OFF + 4);

  const int split = int(blockIdx.x), bh = int(blockIdx.y);
  const int b = bh / p.H;
  int kv_len = p.Nkv;
  if (p.key_lens != nullptr) kv_len = min(kv_len, max(p.key_lens[b], 0));
  // the keys of this split below the cache length
  const int c0 = split * p.chunk;
  const int c1 = min(c0 + p.chunk, kv_len);
  const int n_blk = c1 > c0 ? (c1 - c0 + 127) / 128 : 0;

  if (tid == 0) {
    mbar_init(q_full, 1);
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
      mbar_init(&s_free[s], 4);
      mbar_init(&p_full[s], 4);
    }
    mbar_init(pv_done, 1);
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
  // the combine kernel (a programmatic dependent launch) may be scheduled from here on; it waits
  // for this whole grid before it reads anything
  asm volatile("griddepcontrol.launch_dependents;");

  if (warp == 4) {
    // =========================================================== producer
    if (lane == 0 && n_blk > 0) {
      prefetch_tmap(&tm_q);
      prefetch_tmap(&tm_k);
      prefetch_tmap(&tm_v);
      // Q into tile rows 0-63 and again into rows 64-127 (the 128-byte swizzle repeats every 8 rows,
      // so the second copy sits at the same phase)
      mbar_arrive_expect_tx(q_full, L::TILE);
#pragma unroll
      for (int c = 0; c < D / 64; ++c) {
        tma_load_3d(smem + L::Q_OFF + c * L::SUB, &tm_q, q_full, c * 64, 0, bh);
        tma_load_3d(smem + L::Q_OFF + c * L::SUB + L::QHALF, &tm_q, q_full, c * 64, 0, bh);
      }
      int gk = 0, gv = 0;
      bool ok = true;
      for (int j = 0; ok && j < n_blk; ++j) {
        const int key0 = c0 + j * 128;
        // K_j, then V_j (V is needed one block later than K)
        if (gk >= KST && !mbar_wait(&k_empty[gk % KST], ((gk / KST) - 1) & 1, wc)) { ok = false; break; }
        mbar_arrive_expect_tx(&k_full[gk % KST], L::TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::K_OFF + (gk % KST) * L::TILE + c * L::SUB, &tm_k, &k_full[gk % KST], c * 64, key0, bh);
        ++gk;
        if (gv >= VST && !mbar_wait(&v_empty[gv % VST], ((gv / VST) - 1) & 1, wc)) { ok = false; break; }
        mbar_arrive_expect_tx(&v_full[gv % VST], L::TILE);
#pragma unroll
        for (int c = 0; c < D / 64; ++c)
          tma_load_3d(smem + L::V_OFF + (gv % VST) * L::TILE + c * L::SUB, &tm_v, &v_full[gv % VST], c * 64, key0, bh);
        ++gv;
      }
      // every copy started here lands before the CTA releases its shared memory
      mbar_drain(q_full, 0, p.wait_ns);
      for (int j = max(0, gk - KST); j < gk; ++j) mbar_drain(&k_full[j % KST], (j / KST) & 1, p.wait_ns);
      for (int j = max(0, gv - VST); j < gv; ++j) mbar_drain(&v_full[j % VST], (j / VST) & 1, p.wait_ns);
    }
    __syncwarp();
  } else if (warp == 5) {
    // =========================================================== MMA issuer (whole warp, elect.sync)
    if (n_blk > 0) {
      constexpr uint32_t kIdS = idesc_bf16(128, 128, false, false);   // Q: K-major, K: K-major
      constexpr uint32_t kIdPV = idesc_bf16(128, D, false, true);     // P: TMEM, V: MN-major
      const uint32_t s0 = smem_u32(smem) >> 4;
      constexpr uint32_t kHi = sdesc_sw128_hi(1024), kKM = sdesc_lbo(16), kMN = sdesc_lbo(L::SUB);
      auto wait = [&](uint64_t* bar, uint32_t parity) { return __all_sync(0xffffffffu, mbar_wait(bar, parity, wc)); };
      auto issue_s = [&](int j) {   // S(j) = Q K_j^T into score buffer j % 2
        const uint32_t q_lo = s0 + uint32_t(L::Q_OFF >> 4) + kKM;
        const uint32_t k_lo = s0 + uint32_t((L::K_OFF + (j % KST) * L::TILE) >> 4) + kKM;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {   // 16 features per step: 32 bytes inside a 128-byte row
          const uint32_t off = ((kk >> 2) * L::SUB + (kk & 3) * 32) >> 4;
          mma_ss_elect(tmem + 128 * (j & 1), sdesc_join(q_lo + off, kHi), sdesc_join(k_lo + off, kHi), kIdS,
                      kk > 0 ? 1u : 0u);
        }
        mma_commit_elect(&s_full[j & 1]);
        mma_commit_elect(&k_empty[j % KST]);
      };
      auto issue_pv = [&](int j) {   // O += P(j) V_j   (A = P over the first 64 columns of buffer j % 2)
        const uint32_t v_lo = s0 + uint32_t((L::V_OFF + (j % VST) * L::TILE) >> 4) + kMN;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)   // 16 keys per step: 8 packed TMEM columns, 16 rows of V
          mma_ts_elect(tmem + L::O_COL, tmem + 128 * (j & 1) + kk * 8, sdesc_join(v_lo + kk * (2048 >> 4), kHi),
                      kIdPV, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit_elect(&v_empty[j % VST]);
        mma_commit_elect(pv_done);
      };
      bool ok = wait(q_full, 0);
      for (int j = 0; ok && j <= n_blk; ++j) {
        if (j < n_blk) {
          // buffer j % 2 held S(j-2), read by the softmax, and P(j-2), read by PV(j-2): issued in
          // the previous iteration, so it runs first
          if (j >= 2 && !wait(&s_free[j & 1], ((j - 2) >> 1) & 1)) { ok = false; break; }
          if (!wait(&k_full[j % KST], (j / KST) & 1)) { ok = false; break; }
          tc_fence_after();
          issue_s(j);
        }
        if (j >= 1) {
          const int jp = j - 1;
          if (!wait(&p_full[jp & 1], (jp >> 1) & 1)) { ok = false; break; }
          if (!wait(&v_full[jp % VST], (jp / VST) & 1)) { ok = false; break; }
          tc_fence_after();
          issue_pv(jp);
        }
      }
      mma_commit_elect(fin);
      if (lane == 0) mbar_drain(fin, 0, p.wait_ns);
    }
    __syncwarp();
  } else {
    // =========================================================== softmax (warps 0-3)
    const int r = 32 * warp + lane;       // TMEM lane
    const int half = r >> 6;              // keys [64 half, 64 half + 64) of every block
    const int row = r & 63;               // query row
    const uint32_t lane_base = tmem + (uint32_t(warp * 32) << 16);
    const float sl2 = p.scale_log2;
    const uint64_t sl2x2 = f2_make(sl2, sl2);
    // position of this query in the cache, and the keys it may see
    const int pos = kv_len - p.Nq + row;
    const int lim = row < p.Nq ? (p.causal ? min(kv_len, pos + 1) : kv_len) : 0;   // keys < lim allowed
    float m_ref = -INFINITY, l = 0.f;
    bool ok = true;
    uint32_t zero[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) zero[e] = 0u;
    for (int j = 0; j < n_blk; ++j) {
      const uint32_t sbuf = lane_base + 128 * (j & 1);
      if (!__all_sync(0xffffffffu, mbar_wait(&s_full[j & 1], (j >> 1) & 1, wc))) { ok = false; break; }
      tc_fence_after();
      uint32_t sr[64];
      tmem_ld32(sbuf + 64 * half, *reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      tmem_ld32(sbuf + 64 * half + 32, *reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tmem_ld_wait();
      reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[0]));
      reg_fence32(*reinterpret_cast<uint32_t(*)[32]>(&sr[32]));
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[j & 1]);   // scores read: S(j+2) may follow PV(j)
      const int k0 = c0 + 128 * j + 64 * half;
      if (k0 + 64 > lim) {   // mask keys >= lim
#pragma unroll
        for (int c = 0; c < 64; ++c)
          if (k0 + c >= lim) sr[c] = __float_as_uint(-INFINITY);
      }
      float mx = -INFINITY;
#pragma unroll
      for (int c = 0; c < 64; c += 2) mx = max3f(mx, __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
      const float m_cand = mx * sl2;
      float alpha = 1.f;
      if (m_cand > m_ref + kDecodeRescale) {
        alpha = ex2_approx(m_ref - m_cand);
        m_ref = m_cand;
      }
      // O holds PV up to block j - 1 once that MMA has completed; rescale it if the max moved
      if (j >= 1 && __any_sync(0xffffffffu, alpha != 1.f)) {
        if (!__all_sync(0xffffffffu, mbar_wait(pv_done, (j - 1) & 1, wc))) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int c = 0; c < D / 32; ++c) {
          uint32_t orr[32];
          tmem_ld32(lane_base + L::O_COL + 32 * c, orr);
          tmem_ld_wait();
          reg_fence32(orr);
#pragma unroll
          for (int e = 0; e < 32; ++e) orr[e] = __float_as_uint(__uint_as_float(orr[e]) * alpha);
          tmem_st32(lane_base + L::O_COL + 32 * c, orr);
        }
        tmem_st_wait();
      }
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      const uint64_t negm2 = f2_make(-m_use, -m_use);
      uint64_t rs2 = f2_make(0.f, 0.f);
      uint32_t pk[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const uint64_t x = f2_fma(f2_make(__uint_as_float(sr[2 * e]), __uint_as_float(sr[2 * e + 1])), sl2x2, negm2);
        float x0, x1;
        f2_split(x, x0, x1);
        const uint64_t pp = f2_make(ex2_approx(x0), ex2_approx(x1));
        rs2 = f2_add(rs2, pp);
        float p0, p1;
        f2_split(pp, p0, p1);
        pk[e] = pack_bf16x2(p0, p1);
      }
      // P over the first 64 columns of the buffer (scores already read): this half's 64 keys and
      // zeros for the other half (its query's other row holds those)
      tmem_st32(sbuf + 32 * half, pk);
      tmem_st32(sbuf + 32 * (1 - half), zero);
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[j & 1]);
      float rs0, rs1;
      f2_split(rs2, rs0, rs1);
      l = l * alpha + (rs0 + rs1);
    }
    // ---- partial of this key half: unnormalised O, m (log2 domain), l
    const uint64_t part = (uint64_t(bh) * p.n_part + 2 * split + half) * p.Nq + row;
    if (n_blk > 0 && ok && __all_sync(0xffffffffu, mbar_wait(fin, 0, wc))) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < D / 32; ++c) {
        uint32_t orr[32];
        tmem_ld32(lane_base + L::O_COL + 32 * c, orr);
        tmem_ld_wait();
        reg_fence32(orr);
        if (row < p.Nq) {
          float4* dst = reinterpret_cast<float4*>(p.part_o + part * D + 32 * c);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(orr[4 * e]), __uint_as_float(orr[4 * e + 1]),
                                 __uint_as_float(orr[4 * e + 2]), __uint_as_float(orr[4 * e + 3]));
        }
      }
    } else if (n_blk == 0 && row < p.Nq) {
      float4* dst = reinterpret_cast<float4*>(p.part_o + part * D);
#pragma unroll
      for (int e = 0; e < D / 4; ++e) dst[e] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (row < p.Nq) {
      p.part_ml[2 * part] = (l > 0.f) ? m_ref : -INFINITY;
      p.part_ml[2 * part + 1] = l;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, L::TMEM_COLS);
  }
}

// Merge of the partials of one (head, query row) per warp: lanes take D/32 features each.
template <int D>
__global__ void __launch_bounds__(256) fa_decode_combine_kernel(const DecodeParams p) {
  // launched as a programmatic dependent of the split kernel: wait for that grid to complete
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int w = int(blockIdx.x) * 8 + (int(threadIdx.x) >> 5), lane = int(threadIdx.x) & 31;
  const int rows = p.B * p.H * p.Nq;
  if (w >= rows) return;
  const int bh = w / p.Nq, i = w % p.Nq;
  float m_star = -INFINITY;
  for (int s = lane; s < p.n_part; s += 32)
    m_star = fmaxf(m_star, p.part_ml[2 * ((uint64_t(bh) * p.n_part + s) * p.Nq + i)]);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m_star = fmaxf(m_star, __shfl_xor_sync(0xffffffffu, m_star, off));
  constexpr int PER = D / 32;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  float l_star = 0.f;
  if (m_star != -INFINITY) {
    for (int s = 0; s < p.n_part; ++s) {
      const uint64_t part = (uint64_t(bh) * p.n_part + s) * p.Nq + i;
      const float ms = p.part_ml[2 * part];
      if (ms == -INFINITY) continue;
      const float ws = ex2_approx(ms - m_star);
      l_star += ws * p.part_ml[2 * part + 1];
#pragma unroll
      for (int e = 0; e < PER; ++e) acc[e] = fmaf(ws, p.part_o[part * D + e * 32 + lane], acc[e]);
    }
  }
  const float inv = l_star > 0.f ? 1.f / l_star : 0.f;
  __nv_bfloat16* orow = p.o + (uint64_t(bh) * p.Nq + i) * D;
#pragma unroll
  for (int e = 0; e < PER; ++e) orow[e * 32 + lane] = __float2bfloat16_rn(acc[e] * inv);
  if (lane == 0) p.lse[uint64_t(bh) * p.Nq + i] = l_star > 0.f ? (m_star + lg2_approx(l_star)) * kDecodeLn2 : -INFINITY;
}

}  // namespace fa
