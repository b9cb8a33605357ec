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
//   * adds its 8 values of Q, K and V into fp32 running sums, one per level
//     l >= 1, and writes level l's mean (rounded once to bf16) after every p^l
//     tokens;
//   * sums its 8 squares of Q and of K in fp64; the d/8 lanes of the row then
//     combine their partial sums with xor shuffles (bf16 squares are exact in
//     fp64, so the sum is the exact one whenever the row's magnitudes span
//     less than about 2^15, and any rounding it does is 2^-53-relative);
//   * keeps, per level l >= 1, the running max of those squared norms.
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

__device__ __forceinline__ void cp_async16(uint4* dst, const uint4* src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}

__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

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
  extern __shared__ uint4 ring[];          // [kDepth][3][blockDim.x]
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
  auto stage = [&](int t) {  // copy token t's three vectors into slot t mod kDepth
    if (t < W) {
      uint4* dst = mine + (t % kDepth) * 3 * nt;
      const int64_t off = (int64_t)t * HV;
      cp_async16(dst, gq + off);
      cp_async16(dst + nt, gk + off);
      cp_async16(dst + 2 * nt, gv + off);
    }
    cp_async_commit();  // one group per token, empty past the window
  };

  float aq[L > 1 ? L - 1 : 1][8], ak[L > 1 ? L - 1 : 1][8], av[L > 1 ? L - 1 : 1][8];
  double mq[L], mk[L];   // running max squared norms, levels >= 1
  double pq = 0.0, pk = 0.0;   // level-0 squared norms parked until their batch is rooted
  int left[L];           // tokens still to add before level l's entry is complete
  int ent[L];            // index of level l's current entry (P < 2^31)
#pragma unroll
  for (int l = 0; l < L - 1; ++l)
#pragma unroll
    for (int e = 0; e < 8; ++e) aq[l][e] = ak[l][e] = av[l][e] = 0.f;
#pragma unroll
  for (int l = 0; l < L; ++l) {
    mq[l] = mk[l] = 0.0;
    left[l] = (int)D.lvl_span[l];
    ent[l] = (int)(t0 / D.lvl_span[l]);
  }
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

#pragma unroll
  for (int s = 0; s < kDepth - 1; ++s) stage(s);
#pragma unroll 1
  for (int t = 0; t < W; ++t) {
    // slot (t - 1) mod kDepth was read and used in the previous iteration
    stage(t + kDepth - 1);
    cp_async_wait<kDepth - 1>();   // token t's group has landed
    const uint4* src = mine + (t % kDepth) * 3 * nt;
    const uint4 uq = src[0], uk = src[nt], uv = src[2 * nt];
    const uint32_t wq[4] = {uq.x, uq.y, uq.z, uq.w};
    const uint32_t wk[4] = {uk.x, uk.y, uk.z, uk.w};
    const uint32_t wv[4] = {uv.x, uv.y, uv.z, uv.w};
    float xq[8], xk[8], xv[8];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float2 a = unpack_bf16x2(wq[e]), c = unpack_bf16x2(wk[e]), g = unpack_bf16x2(wv[e]);
      xq[2 * e] = a.x; xq[2 * e + 1] = a.y;
      xk[2 * e] = c.x; xk[2 * e + 1] = c.y;
      xv[2 * e] = g.x; xv[2 * e + 1] = g.y;
    }
    // squares summed as a tree (each product is exact in fp64)
    double sq, sk;
    {
      double tq[4], tk[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const double a0 = xq[2 * e], a1 = xq[2 * e + 1], c0 = xk[2 * e], c1 = xk[2 * e + 1];
        tq[e] = __fma_rn(a0, a0, a1 * a1);
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
#pragma unroll
    for (int l = 1; l < L; ++l) {
      mq[l] = fmax(mq[l], sq);
      mk[l] = fmax(mk[l], sk);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        aq[l - 1][e] += xq[e];
        ak[l - 1][e] += xk[e];
        av[l - 1][e] += xv[e];
      }
      if (--left[l] == 0) {
        const int i = ent[l]++;
        left[l] = (int)D.lvl_span[l];
        const float fs = (float)D.lvl_span[l];
        // x / p^l; for a power-of-two span the product with the exact
        // reciprocal is the same correctly rounded quotient
        const bool pow2 = (D.lvl_span[l] & (D.lvl_span[l] - 1)) == 0;
        const float inv = 1.f / fs;
        auto mean = [&](float x) { return pow2 ? x * inv : __fdiv_rn(x, fs); };
        uint4 oq, ok, ov;
        uint32_t* po = &oq.x; uint32_t* pk2 = &ok.x; uint32_t* pv = &ov.x;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          po[e] = pack_bf16x2(mean(aq[l - 1][2 * e]), mean(aq[l - 1][2 * e + 1]));
          pk2[e] = pack_bf16x2(mean(ak[l - 1][2 * e]), mean(ak[l - 1][2 * e + 1]));
          pv[e] = pack_bf16x2(mean(av[l - 1][2 * e]), mean(av[l - 1][2 * e + 1]));
        }
        const int64_t orow = ((int64_t)D.B * D.pool_row[l] + (int64_t)b * D.lvl_size[l] + i) * HV + j;
        q_lv[orow] = oq;
        k_lv[orow] = ok;
        v_lv[orow] = ov;
#pragma unroll
        for (int e = 0; e < 8; ++e) aq[l - 1][e] = ak[l - 1][e] = av[l - 1][e] = 0.f;
        if (cv == 0) {
          qk_row[D.lvl_off[l] + i] = root_score(mq[l]);
          kq_row[D.lvl_off[l] + i] = root_score(mk[l]);
        }
        mq[l] = mk[l] = 0.0;
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
  const size_t smem = (size_t)kDepth * 3 * threads * sizeof(uint4);   // 48 KB
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
