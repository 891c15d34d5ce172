// fp32 attention forward on the CUDA cores (FFMA, no TF32: a 10-bit-mantissa tensor-core path
// cannot meet a 1e-5 absolute bar).  Same semantics as the bf16 path: online softmax over key
// tiles held in shared memory ("48 FlashAttention", block "Tiling и online softmax"), causal and
// key-padding masks, counter-hash dropout, lse = m + ln l.
//
// Also the dropout-mask kernel that writes the keep decisions of the counter hash, so that a
// test can compare them bit for bit with an independent implementation.
#pragma once
#include "dropout_hash.cuh"

namespace fa {

struct F32Params {
  const float* q;
  const float* k;
  const float* v;
  float* o;
  float* lse;
  const int32_t* key_lens;
  int B, H, N;
  int d;                       // head dimension, 1..128
  int causal;
  float scale;
  int dropout;
  uint32_t drop_thr;
  float drop_scale;
  uint64_t seed;
};

// Two threads per query row (64 rows per CTA of 128 threads), each holding half of the row's
// DP/2 features of q and of the output accumulator; the dot product of a key is the sum of the two
// halves (one shuffle).  DP is the head dimension rounded up to a multiple of 32; features d..DP-1
// read as zero and are not written.  K and V are staged in shared memory 32 keys at a time.
template <int DP>
__global__ void __launch_bounds__(128) fa_fwd_f32_kernel(const F32Params p) {
  constexpr int KT = 32, HALF = DP / 2, ROWS = 64;
  __shared__ float ks[KT][DP];
  __shared__ float vs[KT][DP];
  const int d = p.d;
  const int bh = blockIdx.y;
  const int b = bh / p.H;
  const int half = threadIdx.x & 1;
  const int row = blockIdx.x * ROWS + (threadIdx.x >> 1);
  const bool valid = row < p.N;
  const uint64_t base = uint64_t(bh) * p.N;
  int kv_end = p.N;
  if (p.key_lens != nullptr) kv_end = min(kv_end, max(p.key_lens[b], 0));
  int kv_stop = kv_end;
  if (p.causal) kv_stop = min(kv_stop, int(blockIdx.x) * ROWS + ROWS);

  float qr[HALF], acc[HALF];
#pragma unroll
  for (int c = 0; c < HALF; ++c) {
    const int f = half * HALF + c;
    qr[c] = (valid && f < d) ? p.q[(base + row) * d + f] : 0.f;
    acc[c] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int j0 = 0; j0 < kv_stop; j0 += KT) {
    __syncthreads();
    for (int e = threadIdx.x; e < KT * DP; e += 128) {
      const int jj = e / DP, c = e % DP;
      const int j = j0 + jj;
      const bool in = j < p.N && c < d;
      ks[jj][c] = in ? p.k[(base + j) * d + c] : 0.f;
      vs[jj][c] = in ? p.v[(base + j) * d + c] : 0.f;
    }
    __syncthreads();
    for (int jj = 0; jj < KT; ++jj) {
      const int j = j0 + jj;
      float s = 0.f;
#pragma unroll
      for (int c = 0; c < HALF; ++c) s = fmaf(qr[c], ks[jj][half * HALF + c], s);
      s += __shfl_xor_sync(0xffffffffu, s, 1);   // the other half of the row's features
      if (j >= kv_end || (p.causal && j > row)) continue;
      s *= p.scale;
      if (s > m) {
        const float alpha = expf(m - s);
        l *= alpha;
#pragma unroll
        for (int c = 0; c < HALF; ++c) acc[c] *= alpha;
        m = s;
      }
      float pr = expf(s - m);
      l += pr;
      if (p.dropout) {
        pr = dropout_keep(p.seed, base + uint64_t(row), dropout_row_draws(p.N), j, p.drop_thr) ? pr * p.drop_scale : 0.f;
      }
#pragma unroll
      for (int c = 0; c < HALF; ++c) acc[c] = fmaf(pr, vs[jj][half * HALF + c], acc[c]);
    }
  }
  if (valid) {
    const float inv = l > 0.f ? 1.f / l : 0.f;
#pragma unroll
    for (int c = 0; c < HALF; ++c) {
      const int f = half * HALF + c;
      if (f < d) p.o[(base + row) * d + f] = acc[c] * inv;
    }
    if (half == 0) p.lse[base + row] = l > 0.f ? m + logf(l) : -INFINITY;
  }
}

__global__ void __launch_bounds__(256) fa_dropout_mask_kernel(uint8_t* keep, uint64_t total, int N, uint64_t seed,
                                                              uint32_t thr) {
  const uint64_t W = dropout_row_draws(N);
  for (uint64_t i = uint64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += uint64_t(gridDim.x) * blockDim.x)
    keep[i] = dropout_keep(seed, i / uint64_t(N), W, int(i % uint64_t(N)), thr) ? 1 : 0;
}

}  // namespace fa
