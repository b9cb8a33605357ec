// Stage (i) and the scores of stage (ii) of Lighthouse Attention in one pass
// over Q, K and V ("Long Context Pre-Training with Lighthouse Attention",
// Sec. 3.3 pyramid and Sec. 3.4 scoring).
//
// One thread owns one 16-byte vector (8 features) of one (token, head) row
// and walks the W = p^(L-1) tokens of one coarsest window.  Consecutive
// threads own consecutive vectors of a token row, so every warp-wide copy is
// 512 contiguous bytes.  The thread streams its vectors of Q, K and V through
// a private ring of kDepth token slots in shared memory (cp.async, 16 bytes
// per copy): up to kDepth - 1 tokens are in flight while it works on the
// current one, and as each thread reads only what it copied itself, no block
// barrier is needed.  Per token the thread:
//   * adds its 8 values of Q, K and V into the fp32 sums of the current
//     level-1 entry; when an entry of level l completes, its mean (sum / p^l,
//     rounded once to bf16) is written and its sums are added into level
//     l+1's, which are kept in the thread's own shared-memory slots (so a
//     level-l sum is the fp32 sum of its p children's sums);
//   * sums its 8 squares of Q and of K in fp64; the d/8 lanes of the row then
//     combine their partial sums with xor shuffles (bf16 squares are exact in
//     fp64, so the sum is the exact one whenever the row's magnitudes span
//     less than about 2^15, and any rounding it does is 2^-53-relative);
//   * keeps the running max of those squared norms for the current level-1
//     entry, folded upwards the same way.
// A score is the fp64 square root of a squared norm, rounded once to fp32; a
// coarse score is the max of the level-0 scores in its window, which is the
// root of the max squared norm, since x -> fp32(sqrt(x)) is monotone, so it
// takes one root per coarse entry.  Level-0 roots are taken in lane batches:
// the squared norm of the window's j-th token waits in lane j mod (d/8) until
// the batch is full, and then every lane of the row takes one root and the
// batch goes out as one contiguous store.
#include "lh_common.cuh"

namespace {

constexpr int kDepth = 4;  // token slots in each thread's ring

__device__ __forceinline__ float root_score(double sq) {
  return __double2float_rn(__dsqrt_rn(sq));
}

template <int L>
__global__ void __launch_bounds__(256, 2) k_pyramid_score(LhDims D, const uint4* __restrict__ q,
                                                       const uint4* __restrict__ k,
                                                       const uint4* __restrict__ v,
                                                       uint4* __restrict__ q_lv,
                                                       uint4* __restrict__ k_lv,
                                                       uint4* __restrict__ v_lv,
                                                       float* __restrict__ qk,
                                                       float* __restrict__ kq) {
  // [kDepth][3][blockDim.x] token ring, then [L-2][6][blockDim.x] float4 level sums
  extern __shared__ uint4 ring[];
  const int V = D.d >> 3;                  // vectors per row (8 or 16)
  const int HV = D.H * V;                  // vectors per token
  const int W = (int)D.lvl_span[L - 1];    // tokens per coarsest window
  const int64_t n_win = D.N / W;
  const int64_t item = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  const int64_t total = (int64_t)D.B * n_win * HV;
  // Row groups (V lanes) are whole because total is a multiple of HV; the
  // shuffles below stay inside a group and name only live lanes.
  const unsigned live = __ballot_sync(0xffffffffu, item < total);
  if (item >= total) return;
  const int j = (int)(item % HV);
  const int64_t bw = item / HV;
  const int b = (int)(bw / n_win);
  const int64_t win = bw % n_win;
  const int h = j / V;
  const int cv = j % V;
  const int64_t t0 = win * W;
  const int64_t bh = (int64_t)b * D.H + h;
  float* qk_row = qk + bh * D.P;
  float* kq_row = kq + bh * D.P;

  const int64_t row0 = ((int64_t)b * D.N + t0) * HV + j;   // vector index of token t0
  const uint4* gq = q + row0;
  const uint4* gk = k + row0;
  const uint4* gv = v + row0;
  const unsigned nt = blockDim.x;
  uint4* mine = ring + threadIdx.x;
  float4* sums = reinterpret_cast<float4*>(ring + kDepth * 3 * nt) + threadIdx.x;
  auto stage = [&](int t) {  // copy token t's three vectors into slot t mod kDepth
    if (t < W) {
      uint4* dst = mine + (t % kDepth) * 3 * nt;
      const int64_t off = (int64_t)t * HV;
      lh_cp_async16(dst, gq + off);
      lh_cp_async16(dst + nt, gk + off);
      lh_cp_async16(dst + 2 * nt, gv + off);
    }
    lh_cp_async_commit();  // one group per token, empty past the window
  };

  // Level 1 sums in registers: a1[m][e], m = Q, K, V.  Levels l >= 2 keep
  // theirs in this thread's shared-memory slots sums[((l-2)*6 + c) nt],
  // c = 2m + half; they change only when a level l-1 entry completes.
  float a1[3][8];
#pragma unroll
  for (int m = 0; m < 3; ++m)
#pragma unroll
    for (int e = 0; e < 8; ++e) a1[m][e] = 0.f;
#pragma unroll
  for (int c = 0; c < 6 * (L > 2 ? L - 2 : 0); ++c) sums[c * nt] = make_float4(0.f, 0.f, 0.f, 0.f);
  double mq[L], mk[L];   // running max squared norms of level l's current entry (l >= 1)
  int left[L];           // level l: level-(l-1) entries still to complete (tokens for l = 1)
  int ent[L];            // index of level l's current entry (P < 2^31)
#pragma unroll
  for (int l = 0; l < L; ++l) {
    mq[l] = mk[l] = 0.0;
    left[l] = D.p;
    ent[l] = (int)(t0 / D.lvl_span[l]);
  }
  double pq = 0.0, pk = 0.0;   // level-0 squared norms parked until their batch is rooted
  // Token t is complete with squared norms (sq, sk): park them in lane
  // t mod V, and once the batch is full or the window ends, the batch's lanes
  // write their roots.
  auto settle0 = [&](int t, double sq, double sk) {
    const int pos = t & (V - 1);
    if (pos == cv) {
      pq = sq;
      pk = sk;
    }
    if ((pos == V - 1 || t == W - 1) && cv <= pos) {
      const int64_t e = D.lvl_off[0] + t0 + (t - pos) + cv;
      qk_row[e] = root_score(pq);
      kq_row[e] = root_score(pk);
    }
  };
  // Level l's current entry is complete with fp32 sums s[m][e]: write its
  // mean, rounded once to bf16, and its scores (the roots of the max squared
  // norms; lane 0 of the row).
  auto emit = [&](int l, const float (*s)[8]) {
    const int i = ent[l]++;
    const float fs = (float)D.lvl_span[l];
    // x / p^l; for a power-of-two span the product with the exact
    // reciprocal is the same correctly rounded quotient
    const bool pow2 = (D.lvl_span[l] & (D.lvl_span[l] - 1)) == 0;
    const float inv = 1.f / fs;
    auto mean = [&](float x) { return pow2 ? x * inv : __fdiv_rn(x, fs); };
    uint4 o[3];
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      o[m].x = pack_bf16x2(mean(s[m][0]), mean(s[m][1]));
      o[m].y = pack_bf16x2(mean(s[m][2]), mean(s[m][3]));
      o[m].z = pack_bf16x2(mean(s[m][4]), mean(s[m][5]));
      o[m].w = pack_bf16x2(mean(s[m][6]), mean(s[m][7]));
    }
    const int64_t orow = ((int64_t)D.B * D.pool_row[l] + (int64_t)b * D.lvl_size[l] + i) * HV + j;
    q_lv[orow] = o[0];
    k_lv[orow] = o[1];
    v_lv[orow] = o[2];
    if (cv == 0) {
      qk_row[D.lvl_off[l] + i] = root_score(mq[l]);
      kq_row[D.lvl_off[l] + i] = root_score(mk[l]);
    }
  };
  // Add a completed level-(l-1) entry's sums into level l's slots.
  auto fold = [&](int l, const float (*s)[8]) {
#pragma unroll
    for (int c = 0; c < 6; ++c) {
      float4 a = sums[((l - 2) * 6 + c) * nt];
      const float* x = &s[c >> 1][(c & 1) * 4];
      a.x += x[0]; a.y += x[1]; a.z += x[2]; a.w += x[3];
      sums[((l - 2) * 6 + c) * nt] = a;
    }
  };

#pragma unroll
  for (int s = 0; s < kDepth - 1; ++s) stage(s);
#pragma unroll 1
  for (int t = 0; t < W; ++t) {
    // slot (t - 1) mod kDepth was read and used in the previous iteration
    stage(t + kDepth - 1);
    lh_cp_async_wait<kDepth - 1>();   // token t's group has landed
    const uint4* src = mine + (t % kDepth) * 3 * nt;
    const uint4 u[3] = {src[0], src[nt], src[2 * nt]};
    float x[3][8];
#pragma unroll
    for (int m = 0; m < 3; ++m) {
      const uint32_t w[4] = {u[m].x, u[m].y, u[m].z, u[m].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float2 f = unpack_bf16x2(w[e]);
        x[m][2 * e] = f.x;
        x[m][2 * e + 1] = f.y;
      }
    }
    // squares summed as a tree (each product is exact in fp64)
    double sq, sk;
    {
      double tq[4], tk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const double a0 = x[0][2 * e], a1_ = x[0][2 * e + 1], c0 = x[1][2 * e], c1 = x[1][2 * e + 1];
        tq[e] = __fma_rn(a0, a0, a1_ * a1_);
        tk[e] = __fma_rn(c0, c0, c1 * c1);
      }
      sq = (tq[0] + tq[1]) + (tq[2] + tq[3]);
      sk = (tk[0] + tk[1]) + (tk[2] + tk[3]);
    }
    for (int o = V >> 1; o > 0; o >>= 1) {
      sq += __shfl_xor_sync(live, sq, o);
      sk += __shfl_xor_sync(live, sk, o);
    }
    settle0(t, sq, sk);
    if constexpr (L > 1) {
      mq[1] = fmax(mq[1], sq);
      mk[1] = fmax(mk[1], sk);
#pragma unroll
      for (int m = 0; m < 3; ++m)
#pragma unroll
        for (int e = 0; e < 8; ++e) a1[m][e] += x[m][e];
      if (--left[1] == 0) {
        left[1] = D.p;
        emit(1, a1);
        if constexpr (L > 2) {
          fold(2, a1);
          mq[2] = fmax(mq[2], mq[1]);
          mk[2] = fmax(mk[2], mk[1]);
        }
#pragma unroll
        for (int m = 0; m < 3; ++m)
#pragma unroll
          for (int e = 0; e < 8; ++e) a1[m][e] = 0.f;
        mq[1] = mk[1] = 0.0;
        // spans are nested: level l completes only when level l-1 just did
#pragma unroll
        for (int l = 2; l < L; ++l) {
          if (--left[l] != 0) break;
          left[l] = D.p;
          float s[3][8];
#pragma unroll
          for (int c = 0; c < 6; ++c) {
            const float4 a = sums[((l - 2) * 6 + c) * nt];
            float* y = &s[c >> 1][(c & 1) * 4];
            y[0] = a.x; y[1] = a.y; y[2] = a.z; y[3] = a.w;
            sums[((l - 2) * 6 + c) * nt] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
          emit(l, s);
          if (l + 1 < L) {
            fold(l + 1, s);
            mq[l + 1] = fmax(mq[l + 1], mq[l]);
            mk[l + 1] = fmax(mk[l + 1], mk[l]);
          }
          mq[l] = mk[l] = 0.0;
        }
      }
    }
  }
}

template <int L>
cudaError_t launch_L(const LhDims& D, const lh_bf16* q, const lh_bf16* k, const lh_bf16* v,
                     lh_bf16* q_lv, lh_bf16* k_lv, lh_bf16* v_lv, float* qk, float* kq,
                     cudaStream_t st) {
  const int64_t HV = (int64_t)D.H * (D.d >> 3);
  const int64_t total = (int64_t)D.B * (D.N / D.lvl_span[L - 1]) * HV;
  const int threads = 256;
  // 48 KB of token ring plus 24 KB of level sums per level l >= 2
  const size_t smem = (size_t)kDepth * 3 * threads * sizeof(uint4) +
                      (size_t)(L > 2 ? L - 2 : 0) * 6 * threads * sizeof(float4);
  cudaError_t e = cudaFuncSetAttribute(k_pyramid_score<L>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int64_t blocks = (total + threads - 1) / threads;
  k_pyramid_score<L><<<(unsigned)blocks, threads, smem, st>>>(
      D, reinterpret_cast<const uint4*>(q), reinterpret_cast<const uint4*>(k),
      reinterpret_cast<const uint4*>(v), reinterpret_cast<uint4*>(q_lv),
      reinterpret_cast<uint4*>(k_lv), reinterpret_cast<uint4*>(v_lv), qk, kq);
  return cudaGetLastError();
}

}  // namespace

cudaError_t lh_launch_pyramid(const LhDims& D, const lh_bf16* q, const lh_bf16* k,
                              const lh_bf16* v, lh_bf16* q_lv, lh_bf16* k_lv, lh_bf16* v_lv,
                              float* qk, float* kq, cudaStream_t st) {
  switch (D.L) {
    case 1: return launch_L<1>(D, q, k, v, q_lv, k_lv, v_lv, qk, kq, st);
    case 2: return launch_L<2>(D, q, k, v, q_lv, k_lv, v_lv, qk, kq, st);
    case 3: return launch_L<3>(D, q, k, v, q_lv, k_lv, v_lv, qk, kq, st);
    case 4: return launch_L<4>(D, q, k, v, q_lv, k_lv, v_lv, qk, kq, st);
    case 5: return launch_L<5>(D, q, k, v, q_lv, k_lv, v_lv, qk, kq, st);
    case 6: return launch_L<6>(D, q, k, v, q_lv, k_lv, v_lv, qk, kq, st);
    default: return cudaErrorInvalidValue;
  }
}
