// Stage (iii) of Lighthouse Attention: dense causal softmax attention over
// the gathered sub-sequence ("Long Context Pre-Training with Lighthouse
// Attention", Sec. 3.5, Eq. 9).  Because the gather is topologically sorted,
// the mask is the plain S x S causal one, so this is a causal attention
// forward on [BH, S, d] bf16 tensors, written for the sm_100a tensor cores.
//
// One CTA owns two neighbouring tiles of 128 query rows of one (b, h), tile
// a = 2 i and tile b = 2 i + 1, and walks the key/value tiles of 128 rows up
// to b's diagonal; each K / V tile is loaded once for both query tiles.
// Warp roles:
//   warp 0     TMA producer: both Q tiles once, then K and V tiles into
//              their rings;
//   warp 1     MMA issuer, in this order per key tile j:
//                O_a += P_a(j) V(j), S_a(j + 1) = Q_a K(j + 1)^T,
//                O_b += P_b(j) V(j), S_b(j + 1) = Q_b K(j + 1)^T,
//              P read from TMEM (A operand in tensor memory), everything
//              else from shared memory;
//   warps 2-5  softmax warpgroup of tile a, warps 6-9 of tile b: one query
//              row per thread (TMEM lane = row), all 128 columns of each
//              score tile, exact running max and row sum.
// Each warpgroup's softmax of tile j runs while the tensor pipe works for
// the other tile, so the two warpgroups take turns (ping-pong) and each
// sub-partition always has one softmax warp with work.  Because the issuer
// commits S_x(j + 1) after P_x(j) V(j), a finished S_x(j + 1) also means
// that O_x holds every earlier product: the softmax rescales O_x for the
// new running max with no further wait.
//
// TMEM (512 columns, one CTA per SM): S_a 0..127 and S_b 128..255 (P_x as
// packed bf16 over the first 64 columns of S_x), O_a from 256, O_b from
// 256 + d.  Shared memory: Q_a, Q_b, KST K stages and VST V stages (128 x d
// bf16 each), 128-byte swizzled, 1024-byte aligned.
//
// Blocks of a ring (context parallelism, the pages' multi-GPU training
// note: the gathered sub-sequences of consecutive shards rotate through
// ring attention).  The same kernel computes one step of it: the rows of
// one shard's sub-sequence against one K/V block of the same length S,
// either the shard's own block (causal, as above) or an earlier shard's
// block (`full`: every key visible; keys past S masked).  Partial results
// merge by log-sum-exp into fp32 accumulators, in base 2:
//   lse2 = log2(2^u + 2^w),  O = O_u 2^(u - lse2) + O_w 2^(w - lse2)
// with u the accumulated and w this block's lse2, and O_u, O_w their
// normalised outputs.
// `first` writes the accumulators without reading them; `last` writes the
// bf16 output and natural-log LSE instead of them.  first && last is the
// plain single-block attention.
#include <cudaTypedefs.h>

#include <type_traits>

#include "lh_sm100.cuh"

namespace {

using namespace sm100;

constexpr int BM = 128;
constexpr int BN = 128;
constexpr int KST = 3;
constexpr int VST = 2;
constexpr int kThreads = 320;
constexpr int kWG = 128;             // threads of one softmax warpgroup
constexpr uint32_t kTmemCols = 512;

template <int HD>
struct FwdLayout {
  static constexpr uint32_t q = 0;                        // Q_a, Q_b
  static constexpr uint32_t k = q + 2 * BM * HD * 2;
  static constexpr uint32_t v = k + KST * BN * HD * 2;
  static constexpr uint32_t bar = v + VST * BN * HD * 2;
  static constexpr uint32_t bytes = bar + 256;
};

// At least half the shared memory of an SM: one CTA per SM, since each
// allocates all 512 TMEM columns.
constexpr uint32_t kSmemBytes = FwdLayout<128>::bytes + 1024;
static_assert(kSmemBytes > 232448 / 2 && kSmemBytes <= 232448, "one CTA per SM");
static_assert(FwdLayout<64>::bytes <= kSmemBytes, "d = 64 fits the same launch");

struct Bars {
  // sfull[x] / pfull[x] complete once per key tile of query tile x; neither
  // side can run two phases ahead, since each waits for the other's last.
  uint64_t qfull;
  uint64_t kfull[KST], kempty[KST], vfull[VST], vempty[VST];
  uint64_t sfull[2], pfull[2], odone[2];
  uint32_t tmem_base;
};
static_assert(sizeof(Bars) <= 256, "barrier block");

template <int HD>
__global__ void __launch_bounds__(kThreads, 1)
    k_attn_fwd(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, uint4* __restrict__ og,
               uint4* __restrict__ og_lo, float* __restrict__ lse, int S, int BH,
               float scale_log2, int* status, int full, int first, int last,
               float* __restrict__ o_acc, float* __restrict__ lse2_acc) {
  using Lay = FwdLayout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  Bars* bars = reinterpret_cast<Bars*>(smem + Lay::bar);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int n_qt = (S + BM - 1) / BM;
  const int n_pr = (n_qt + 1) / 2;
  const int qa = 2 * (n_pr - 1 - (int)(blockIdx.x / BH));  // longest rows first
  const int bh = (int)(blockIdx.x % BH);
  const bool has_b = qa + 1 < n_qt;
  // key tiles walked by each query tile: up to its diagonal (BN == BM), or
  // all of them for an earlier block; tile b may lie past S (odd tile count)
  const int n_a = full ? n_qt : qa + 1;
  const int n_b = has_b ? (full ? n_qt : qa + 2) : 0;
  const int n_kv = n_a > n_b ? n_a : n_b;

  if (threadIdx.x == 0) {
    mbar_init(&bars->qfull, 1);
    for (int s = 0; s < KST; ++s) {
      mbar_init(&bars->kfull[s], 1);
      mbar_init(&bars->kempty[s], 1);
    }
    for (int s = 0; s < VST; ++s) {
      mbar_init(&bars->vfull[s], 1);
      mbar_init(&bars->vempty[s], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&bars->sfull[x], 1);
      mbar_init(&bars->pfull[x], kWG);
      mbar_init(&bars->odone[x], 1);
    }
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bars->tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bars->tmem_base;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&tmQ);
      tma_prefetch_desc(&tmK);
      tma_prefetch_desc(&tmV);
      const int nq = has_b ? 2 : 1;
      mbar_expect_tx(&bars->qfull, nq * BM * HD * 2);
      for (int x = 0; x < nq; ++x)
        for (int blk = 0; blk < HD / 64; ++blk)
          tma_load_3d(&tmQ, &bars->qfull, smem + Lay::q + x * BM * HD * 2 + blk * BM * 128,
                      64 * blk, (qa + x) * BM, bh);
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % KST, t = j % VST;
        if (!mbar_wait(&bars->kempty[s], ((j / KST) & 1) ^ 1, status, 1)) break;
        mbar_expect_tx(&bars->kfull[s], BN * HD * 2);
        for (int blk = 0; blk < HD / 64; ++blk)
          tma_load_3d(&tmK, &bars->kfull[s], smem + Lay::k + s * BN * HD * 2 + blk * BN * 128,
                      64 * blk, j * BN, bh);
        if (!mbar_wait(&bars->vempty[t], ((j / VST) & 1) ^ 1, status, 2)) break;
        mbar_expect_tx(&bars->vfull[t], BN * HD * 2);
        for (int blk = 0; blk < HD / 64; ++blk)
          tma_load_3d(&tmV, &bars->vfull[t], smem + Lay::v + t * BN * HD * 2 + blk * BN * 128,
                      64 * blk, j * BN, bh);
      }
    }
  } else if (warp == 1) {
    // MMA issuer (whole-warp loop, one lane issues).
    constexpr uint32_t idS = idesc_bf16(BM, BN, 0, 0);
    constexpr uint32_t idO = idesc_bf16(BM, HD, 0, 1);
    const uint32_t sQ = smem_u32(smem + Lay::q), sK = smem_u32(smem + Lay::k);
    const uint32_t sV = smem_u32(smem + Lay::v);
    auto score = [&](int x, int j) {   // S_x(j) = Q_x K(j)^T into columns 128 x
      const uint32_t qb = sQ + x * BM * HD * 2, kb = sK + (j % KST) * BN * HD * 2;
#pragma unroll
      for (int ks = 0; ks < HD / 16; ++ks) {
        const uint32_t off = (ks >> 2) * BM * 128 + (ks & 3) * 32;   // BM == BN
        mma_bf16_w(tmem + x * BN, sdesc_sw128(qb + off, 16, 1024), sdesc_sw128(kb + off, 16, 1024),
                   idS, ks > 0 ? 1u : 0u);
      }
      mma_commit_w(&bars->sfull[x]);
    };
    bool ok = mbar_wait_w(&bars->qfull, 0, status, 3) && mbar_wait_w(&bars->kfull[0], 0, status, 4);
    if (ok) {
      tc_fence_after();
      score(0, 0);
      if (n_b > 0) score(1, 0);
      mma_commit_w(&bars->kempty[0]);
    }
    for (int j = 0; ok && j < n_kv; ++j) {
      const int t = j % VST, s1 = (j + 1) % KST;
      if (!mbar_wait_w(&bars->vfull[t], (j / VST) & 1, status, 6)) break;
      bool k_ready = false;
      const uint32_t vb = sV + t * BN * HD * 2;
#pragma unroll
      for (int x = 0; x < 2; ++x) {
        const int nx = x ? n_b : n_a;
        if (j >= nx) continue;
        if (!mbar_wait_w(&bars->pfull[x], j & 1, status, 7)) { ok = false; break; }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < BN / 16; ++ks)
          mma_bf16_ts_w(tmem + 256 + x * HD, tmem + x * BN + ks * 8,
                        sdesc_sw128(vb + ks * 16 * 128, BN * 128, 1024), idO,
                        (j > 0 || ks > 0) ? 1u : 0u);
        if (j + 1 < nx) {
          if (!k_ready && !mbar_wait_w(&bars->kfull[s1], ((j + 1) / KST) & 1, status, 5)) {
            ok = false;
            break;
          }
          k_ready = true;
          tc_fence_after();
          score(x, j + 1);
        } else {
          mma_commit_w(&bars->odone[x]);
        }
      }
      if (!ok) break;
      mma_commit_w(&bars->vempty[t]);
      if (k_ready) mma_commit_w(&bars->kempty[s1]);
    }
  } else {
    // softmax warpgroup x (warps 2-5: tile a, 6-9: tile b); TMEM lane
    // quarter = warp % 4.  Waits are warp-wide (the vote below needs every
    // lane).
    const int x = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int r = quarter * 32 + lane;       // row in the tile = TMEM lane
    const int qt = qa + x;
    const int qrow = qt * BM + r;            // row in the sequence
    const int nx = x ? n_b : n_a;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const uint32_t tS = tmem + lane_addr + x * BN;
    const uint32_t tO = tmem + lane_addr + 256 + x * HD;
    float m_used = -INFINITY, lsum = 0.f;
    bool ok = nx > 0;
    for (int j = 0; ok && j < nx; ++j) {
      if (!mbar_wait_w(&bars->sfull[x], j & 1, status, 8)) { ok = false; break; }
      tc_fence_after();
      uint32_t s[BN];
#pragma unroll
      for (int c = 0; c < BN / 32; ++c)
        tmem_ld32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&s[c * 32]));
      tmem_ld_wait();
      // masked tile: the diagonal (keys <= r) or, for an earlier block, the
      // ragged last tile (keys < S); columns e < lim are kept
      const bool diag = !full && (j == qt);
      const bool msk = diag || (full && (j + 1) * BN > S);
      const int lim = diag ? r + 1 : S - j * BN;
      float mxv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) mxv[u] = -INFINITY;
      if (msk) {
#pragma unroll
        for (int e = 0; e < BN; ++e)
          if (e < lim) mxv[e & 7] = fmaxf(mxv[e & 7], __uint_as_float(s[e]));
      } else {
#pragma unroll
        for (int e = 0; e < BN; e += 2)
          mxv[(e >> 1) & 7] = fmax3(mxv[(e >> 1) & 7], __uint_as_float(s[e]), __uint_as_float(s[e + 1]));
      }
      const float mx = fmaxf(fmaxf(fmaxf(mxv[0], mxv[1]), fmaxf(mxv[2], mxv[3])),
                             fmaxf(fmaxf(mxv[4], mxv[5]), fmaxf(mxv[6], mxv[7])));
      // Exact running max: the largest term so far gets p = 1, which bf16
      // holds exactly.  (A stale max, as lazy rescaling keeps, would round
      // that dominant term by up to 2^-9, and the error would reach
      // D = rowsum(dO * O) of the backward unscaled.)
      const float m_new = fmaxf(m_used, mx * scale_log2);
      const bool grow = m_new > m_used;
      const float alpha = grow ? ex2(m_used - m_new) : 1.f;
      m_used = m_new;
      const float m_sub = m_used == -INFINITY ? 0.f : m_used;
      // x = s scale - m and the row sum in packed fp32 pairs
      const uint64_t sc2 = f2_pack(scale_log2, scale_log2), nm2 = f2_pack(-m_sub, -m_sub);
      uint64_t rs2[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) rs2[u] = f2_pack(0.f, 0.f);
      // two copies of the loop, so that unmasked tiles (all but one) carry no
      // per-column compare
      auto exp_tile = [&](auto masked) {
#pragma unroll
        for (int c = 0; c < BN / 16; ++c) {
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const int i = c * 16 + e;
            const float2 xx = f2_unpack(f2_fma(f2_pack(__uint_as_float(s[i]), __uint_as_float(s[i + 1])), sc2, nm2));
            float p0 = ex2(xx.x), p1 = ex2(xx.y);
            if constexpr (decltype(masked)::value) {
              p0 = (i < lim) ? p0 : 0.f;
              p1 = (i + 1 < lim) ? p1 : 0.f;
            }
            rs2[(i >> 1) & 3] = f2_add(rs2[(i >> 1) & 3], f2_pack(p0, p1));
            pk[e >> 1] = pack_bf16x2(p0, p1);
          }
          // P of keys 16 c .. 16 c + 15 lands on columns 8 c .. 8 c + 7,
          // whose scores were read above
          tmem_st8(tS + c * 8, pk);
        }
      };
      if (msk) exp_tile(std::true_type{});
      else exp_tile(std::false_type{});
      const float2 ra = f2_unpack(f2_add(rs2[0], rs2[1])), rb = f2_unpack(f2_add(rs2[2], rs2[3]));
      const float rs = (ra.x + ra.y) + (rb.x + rb.y);
      lsum = lsum * alpha + rs;
      // O_x holds P_x V of the earlier tiles (complete: S_x(j) was issued
      // after them); bring it to the new max
      if (j > 0 && __any_sync(0xffffffffu, grow)) {
        const uint64_t a2 = f2_pack(alpha, alpha);
#pragma unroll
        for (int c = 0; c < HD / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(tO + c * 32, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const float2 y = f2_unpack(f2_mul(f2_pack(__uint_as_float(o[e]), __uint_as_float(o[e + 1])), a2));
            o[e] = __float_as_uint(y.x);
            o[e + 1] = __float_as_uint(y.y);
          }
          tmem_st32(tO + c * 32, o);
        }
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->pfull[x]);
    }
    // ---- epilogue: O_x / l and LSE of this tile's rows
    if (ok && mbar_wait_w(&bars->odone[x], 0, status, 10)) {
      tc_fence_after();
      const bool chain = !(first && last);           // a ring step that merges
      const int64_t row_off = (int64_t)bh * S + qrow;
      const float lse2_a = (chain && !first && qrow < S) ? lse2_acc[row_off] : -INFINITY;
      float w = 1.f / lsum;                          // finite: column 0 is never masked
      // ring step: weights of the accumulated and of this block's output
      float lse2_out = m_used + __log2f(lsum), fa = 0.f;
      if (chain) {
        const float b = lse2_out;
        const float mx = fmaxf(lse2_a, b);
        const float wa = first ? 0.f : ex2(lse2_a - mx), wb = ex2(b - mx);
        const float z = wa + wb;
        lse2_out = mx + __log2f(z);
        fa = wa / z;
        w *= wb / z;
      }
#pragma unroll
      for (int c = 0; c < HD / 32; ++c) {            // 32-column chunk of the output
        uint32_t o[32];
        tmem_ld32(tO + c * 32, o);
        tmem_ld_wait();
        if (qrow < S) {
          const int64_t base = ((int64_t)bh * S + qrow) * (HD / 8) + c * 4;
          float4* acc = chain ? reinterpret_cast<float4*>(o_acc) + row_off * (HD / 4) + c * 8
                              : nullptr;
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            float xv[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) xv[e] = __uint_as_float(o[v * 8 + e]) * w;
            if (chain && !first) {
              const float4 a = acc[2 * v], b = acc[2 * v + 1];
              xv[0] += fa * a.x; xv[1] += fa * a.y; xv[2] += fa * a.z; xv[3] += fa * a.w;
              xv[4] += fa * b.x; xv[5] += fa * b.y; xv[6] += fa * b.z; xv[7] += fa * b.w;
            }
            if (!last) {                             // keep the merged fp32 output
              acc[2 * v] = make_float4(xv[0], xv[1], xv[2], xv[3]);
              acc[2 * v + 1] = make_float4(xv[4], xv[5], xv[6], xv[7]);
              continue;
            }
            uint4 wv;
            wv.x = pack_bf16x2(xv[0], xv[1]); wv.y = pack_bf16x2(xv[2], xv[3]);
            wv.z = pack_bf16x2(xv[4], xv[5]); wv.w = pack_bf16x2(xv[6], xv[7]);
            og[base + v] = wv;
            if (og_lo) {
              const uint32_t ww[4] = {wv.x, wv.y, wv.z, wv.w};
              uint32_t rr[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float2 hh = unpack_bf16x2(ww[e]);
                rr[e] = pack_bf16x2(xv[2 * e] - hh.x, xv[2 * e + 1] - hh.y);
              }
              og_lo[base + v] = make_uint4(rr[0], rr[1], rr[2], rr[3]);
            }
          }
        }
      }
      if (qrow < S) {
        if (last) lse[row_off] = lse2_out * 0.69314718055994531f;
        else lse2_acc[row_off] = lse2_out;
      }
    }
    tc_fence_before();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

}  // namespace

// cuTensorMapEncodeTiled from the driver, looked up once.
PFN_cuTensorMapEncodeTiled_v12000 lh_tensormap_encoder() { return get_encode(); }

// Tensor map over a [BH, rows, d] bf16 tensor, box = 64 features x box_rows
// rows of one (b, h), 128-byte swizzle; rows past `rows` read as zero.
bool lh_make_tmap_3d(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int d,
                     int box_rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t dims[3] = {(cuuint64_t)d, (cuuint64_t)rows, (cuuint64_t)BH};
  cuuint64_t strides[2] = {(cuuint64_t)d * 2, (cuuint64_t)rows * d * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

cudaError_t lh_launch_attn_fwd(int BH, int64_t S, int d, float scale, const lh_bf16* qg,
                               const lh_bf16* kg, const lh_bf16* vg, lh_bf16* og,
                               lh_bf16* og_lo, float* lse, int* status, cudaStream_t st,
                               int full, int first, int last, float* o_acc, float* lse2_acc) {
  CUtensorMap tq, tk, tv;
  if (!lh_make_tmap_3d(&tq, qg, BH, S, d, BM) || !lh_make_tmap_3d(&tk, kg, BH, S, d, BN) ||
      !lh_make_tmap_3d(&tv, vg, BH, S, d, BN))
    return cudaErrorInvalidValue;
  const int n_qt = (int)((S + BM - 1) / BM);
  const dim3 grid((unsigned)((n_qt + 1) / 2 * BH));
  const float scale_log2 = scale * 1.4426950408889634f;
  if (d == 128) {
    cudaFuncSetAttribute(k_attn_fwd<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    k_attn_fwd<128><<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, (uint4*)og, (uint4*)og_lo, lse,
                                                         (int)S, BH, scale_log2, status, full,
                                                         first, last, o_acc, lse2_acc);
  } else if (d == 64) {
    cudaFuncSetAttribute(k_attn_fwd<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
    k_attn_fwd<64><<<grid, kThreads, kSmemBytes, st>>>(tq, tk, tv, (uint4*)og, (uint4*)og_lo, lse,
                                                        (int)S, BH, scale_log2, status, full,
                                                        first, last, o_acc, lse2_acc);
  } else {
    return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}
