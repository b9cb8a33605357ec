// Stage (i) and the scores of stage (ii) of Lighthouse Attention in one pass
// over Q, K and V ("Long Context Pre-Training with Lighthouse Attention",
// Sec. 3.3 pyramid and Sec. 3.4 scoring).
//
// One thread owns one 16-byte vector (8 features) of one (token, head) row
// and walks the W = p^(L-1) tokens of one coarsest window.  Consecutive
// threads own consecutive vectors of a token row, so every warp-wide load is
// 512 contiguous bytes.  Per token the thread:
//   * adds its 8 values of Q, K and V into fp32 running sums, one per level
//     l >= 1, and writes level l's mean (rounded once to bf16) after every p^l
//     tokens;
//   * sums its 8 squares of Q and of K in fp64; the d/8 lanes of the row then
//     combine their partial sums with xor shuffles, and the fp64 square root,
//     rounded once to fp32, is the level-0 score (bf16 squares are exact in
//     fp64, so the sum is the exact one whenever the row's magnitudes span
//     less than about 2^15, and any rounding it does is 2^-53-relative);
//   * keeps the running max of the level-0 scores per level: a coarse score
//     is the max of the level-0 scores in its window.
#include "lh_common.cuh"

namespace {

template <int L>
__global__ void __launch_bounds__(256, 2) k_pyramid_score(LhDims D, const uint4* __restrict__ q,
                                                       const uint4* __restrict__ k,
                                                       const uint4* __restrict__ v,
                                                       uint4* __restrict__ q_lv,
                                                       uint4* __restrict__ k_lv,
                                                       uint4* __restrict__ v_lv,
                                                       float* __restrict__ qk,
                                                       float* __restrict__ kq) {
  const int V = D.d >> 3;                  // vectors per row
  const int HV = D.H * V;                  // vectors per token
  const int64_t W = D.lvl_span[L - 1];     // tokens per coarsest window
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

  float aq[L > 1 ? L - 1 : 1][8], ak[L > 1 ? L - 1 : 1][8], av[L > 1 ? L - 1 : 1][8];
  float mq[L], mk[L];
  int left[L];        // tokens still to add before level l's entry is complete
  int64_t ent[L];     // index of level l's current entry
#pragma unroll
  for (int l = 0; l < L - 1; ++l)
#pragma unroll
    for (int e = 0; e < 8; ++e) aq[l][e] = ak[l][e] = av[l][e] = 0.f;
#pragma unroll
  for (int l = 0; l < L; ++l) {
    mq[l] = mk[l] = 0.f;
    left[l] = (int)D.lvl_span[l];
    ent[l] = t0 / D.lvl_span[l];
  }

  const int64_t row0 = ((int64_t)b * D.N + t0) * HV + j;   // vector index of token t0
#pragma unroll 2
  for (int t = 0; t < (int)W; ++t) {
    const int64_t idx = row0 + t * HV;
    const uint4 uq = __ldg(q + idx), uk = __ldg(k + idx), uv = __ldg(v + idx);
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
    double sq = 0.0, sk = 0.0;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      sq = __fma_rn((double)xq[e], (double)xq[e], sq);
      sk = __fma_rn((double)xk[e], (double)xk[e], sk);
    }
    for (int o = V >> 1; o > 0; o >>= 1) {
      sq += __shfl_xor_sync(live, sq, o);
      sk += __shfl_xor_sync(live, sk, o);
    }
    const float nq = __double2float_rn(__dsqrt_rn(sq));
    const float nk = __double2float_rn(__dsqrt_rn(sk));
    const int64_t tok = t0 + t;
    if (cv == 0) {
      qk_row[tok] = nq;
      kq_row[tok] = nk;
    }
#pragma unroll
    for (int l = 1; l < L; ++l) {
      mq[l] = fmaxf(mq[l], nq);
      mk[l] = fmaxf(mk[l], nk);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        aq[l - 1][e] += xq[e];
        ak[l - 1][e] += xk[e];
        av[l - 1][e] += xv[e];
      }
      if (--left[l] == 0) {
        const int64_t i = ent[l]++;
        left[l] = (int)D.lvl_span[l];
        const float fs = (float)D.lvl_span[l];
        // x / p^l; for a power-of-two span the product with the exact
        // reciprocal is the same correctly rounded quotient
        const bool pow2 = (D.lvl_span[l] & (D.lvl_span[l] - 1)) == 0;
        const float inv = 1.f / fs;
        auto mean = [&](float x) { return pow2 ? x * inv : __fdiv_rn(x, fs); };
        uint4 oq, ok, ov;
        uint32_t* pq = &oq.x; uint32_t* pk = &ok.x; uint32_t* pv = &ov.x;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          pq[e] = pack_bf16x2(mean(aq[l - 1][2 * e]), mean(aq[l - 1][2 * e + 1]));
          pk[e] = pack_bf16x2(mean(ak[l - 1][2 * e]), mean(ak[l - 1][2 * e + 1]));
          pv[e] = pack_bf16x2(mean(av[l - 1][2 * e]), mean(av[l - 1][2 * e + 1]));
        }
        const int64_t orow = ((int64_t)D.B * D.pool_row[l] + (int64_t)b * D.lvl_size[l] + i) * HV + j;
        q_lv[orow] = oq;
        k_lv[orow] = ok;
        v_lv[orow] = ov;
#pragma unroll
        for (int e = 0; e < 8; ++e) aq[l - 1][e] = ak[l - 1][e] = av[l - 1][e] = 0.f;
        if (cv == 0) {
          qk_row[D.lvl_off[l] + i] = mq[l];
          kq_row[D.lvl_off[l] + i] = mk[l];
        }
        mq[l] = mk[l] = 0.f;
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
  const int64_t blocks = (total + threads - 1) / threads;
  k_pyramid_score<L><<<(unsigned)blocks, threads, 0, st>>>(
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
