// Backward of the gathered causal attention of Lighthouse Attention ("Long
// Context Pre-Training with Lighthouse Attention", Sec. 3.2: gradients reach
// Q, K, V through the scatter, the attention of Eq. 9 and the gather).
//
// With s = scale q.k, P = softmax rows (rebuilt from the saved LSE),
// dP = dO V^T and D = rowsum(dO * O):  dS = P (dP - D), dV = P^T dO,
// dK = scale dS^T Q, dQ = scale dS K.  Two tcgen05 kernels, neither with
// floating-point atomics, so every gradient is bitwise reproducible:
//
//  k_attn_bwd_dkdv  one CTA per 128 key rows of one (b, h); walks the query
//                   tiles of 128 rows at and after its diagonal.  TMEM holds
//                   S^T, dP^T (P^T, dS^T as bf16 in place) and the dV, dK
//                   accumulators; the gradient MMAs read P^T / dS^T straight
//                   from TMEM.  Two issuer warps (one per MMA stream).
//  k_attn_bwd_dq    one CTA per 128 query rows; walks the key tiles of 128
//                   rows up to its diagonal, recomputing S (two TMEM
//                   buffers) and dP (dS as bf16 in place), and accumulates
//                   dQ in TMEM from TS MMAs.  Two issuer warps.
//
// Warp roles: warp 0 issues TMA loads of the walked tiles, MMA issuer warps
// commit their MMAs to mbarriers, and two softmax warpgroups (8 warps) own
// the TMEM lanes (= the rows of the stationary tile), each warpgroup half of
// the walked tile's columns: they turn scores into P and dS in fp32.  (The
// backward softmax is elementwise given LSE and D, so the two halves need no
// exchange; two warps per SM sub-partition hide each other's latency.)
// The same shared-memory tile of Q, dO or K serves as a K-major operand in
// one MMA and as an MN-major operand in another.
//
// Ring steps (context parallelism: one shard's query rows against one K/V
// block of the same length S, see the forward kernel): `full` walks every
// tile of an earlier shard's block with no mask (rows and keys past S are
// zero-filled by TMA, so they add nothing); the gradients of a block that
// several steps reach are summed in fp32 accumulators (`first` writes them
// without reading, `last` writes the bf16 result instead), in step order,
// so the sums stay bitwise reproducible.
#include <type_traits>

#include "lh_sm100.cuh"

namespace {

using namespace sm100;

// Both kernels: warp 0 TMA, warps 1 and 10 MMA issuers, warps 2-9 two
// softmax warpgroups (warp w owns TMEM lanes 32 (w % 4) .. +31 and half
// (w - 2) / 4 of the walked tile's columns).
constexpr int kSoftmax = 256;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

// One thread's 32 gradient columns x * mul of a ring step: summed with the
// fp32 accumulator (unless first), then kept there (unless last) or written
// as bf16 (last).  acc: 8 float4, out: 4 uint4.
__device__ __forceinline__ void lh_chain_store(const uint32_t (&o)[32], float mul, float4* acc,
                                               uint4* out, int first, int last) {
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    float x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = __uint_as_float(o[v * 8 + e]) * mul;
    if (!first) {
      const float4 a = acc[2 * v], b = acc[2 * v + 1];
      x[0] += a.x; x[1] += a.y; x[2] += a.z; x[3] += a.w;
      x[4] += b.x; x[5] += b.y; x[6] += b.z; x[7] += b.w;
    }
    if (last) {
      out[v] = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                          pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
    } else {
      acc[2 * v] = make_float4(x[0], x[1], x[2], x[3]);
      acc[2 * v + 1] = make_float4(x[4], x[5], x[6], x[7]);
    }
  }
}

// ------------------------------------------------------------------ dK/dV --

constexpr int KV_M = 128;  // stationary key rows
constexpr int Q_N = 128;   // walked query rows per tile
constexpr int QST = 2;     // stages of the walked Q / dO ring

// warp 0 TMA, warp 1 issuer A (S^T, dV), warps 2-9 softmax, warp 10 issuer B
// (dP^T, dK).
constexpr int kThreadsDkdv = 352;

template <int HD>
struct DkdvLayout {
  static constexpr uint32_t k = 0;
  static constexpr uint32_t v = k + KV_M * HD * 2;
  static constexpr uint32_t q = v + KV_M * HD * 2;            // QST stages
  static constexpr uint32_t dO = q + QST * Q_N * HD * 2;      // QST stages
  static constexpr uint32_t kaug = dO + QST * Q_N * HD * 2;   // [128][16] bf16, constant
  static constexpr uint32_t qaug = kaug + KV_M * 32;          // QST x [128][16] bf16
  static constexpr uint32_t oaug = qaug + QST * Q_N * 32;     // QST x [128][16] bf16
  static constexpr uint32_t bar = oaug + QST * Q_N * 32;
  static constexpr uint32_t bytes = bar + 256;
};

struct DkdvBars {
  // sissued[t % 2]: issuer A has issued S^T(t).  Issuer B waits for it before
  // its own MMAs of step t, so the MMAs on the softmax's critical chain (dV,
  // then S^T) enter the tensor pipe first.  Two barriers by parity, because
  // A may run one step ahead of B.
  uint64_t kvfull, qfull[QST], qempty[QST], sfull, dpfull, pready, dsready, sissued[2], done;
  uint32_t tmem_base;
};

// TMEM columns: S^T 0..127 (P^T as packed bf16 over the first 32 columns of
// each warpgroup's 64), dP^T 128..255 (dS^T likewise), dV 256, dK 256 + HD.
//
// LSE and D enter through the tensor core, not through the softmax threads:
// each score MMA gets one more K = 16 step whose A rows are (-1/2, -1/2,
// -1/2, 0, ...) and whose B row for query q holds x_q split into three bf16
// terms (hi + mid + lo = x_q to fp32 precision), both halves of every 32-byte
// row equal, so the extra step adds -x_q exactly (products of bf16 are exact
// in the fp32 accumulator).  With x = LSE / scale the first MMA yields
// s - LSE / scale, so P = exp2(scale log2(e) (s - LSE / scale)); with x = D
// the second yields dP - D.  The softmax threads then read nothing but TMEM:
// shared-memory loads from those threads stall behind the tensor core's
// operand reads.
//
// Per query tile i the tensor pipe runs two independent streams, each from
// its own issuer warp so that a barrier wait in one never drains the pipe:
//   A: dV += P^T(i-1) dO(i-1), then S^T(i) = K Q(i)^T   (waits P(i-1))
//   B: dK += dS^T(i-1) Q(i-1), then dP^T(i) = V dO(i)^T (waits dS(i-1))
// The softmax warpgroups turn S^T(i) into P (fp32 in registers, bf16 into
// TMEM) while stream B runs, then dP^T(i) into dS while stream A runs.  The
// MMAs of one issuer execute in issue order, so S^T(i) overwriting P^T(i-1)
// after the dV MMAs that read it is safe; likewise dP^T(i) after dK.
template <int HD>
__global__ void __launch_bounds__(kThreadsDkdv, 1)
    k_attn_bwd_dkdv(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                    const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                    const float* __restrict__ lse, const float* __restrict__ delta,
                    uint4* __restrict__ dkg, uint4* __restrict__ dvg, int S, int BH, float scale,
                    int* status, int full, int first, int last, float* __restrict__ dk_acc,
                    float* __restrict__ dv_acc) {
  using Lay = DkdvLayout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  DkdvBars* bars = reinterpret_cast<DkdvBars*>(smem + Lay::bar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = (int)(blockIdx.x / BH);  // key tile 0 walks the most query tiles: first
  const int bh = (int)(blockIdx.x % BH);
  const int n_q = (S + Q_N - 1) / Q_N;
  const int i0 = full ? 0 : kt;            // the diagonal query tile (Q_N == KV_M)
  const int n_it = n_q - i0;

  if (threadIdx.x == 0) {
    mbar_init(&bars->kvfull, 1);
    for (int s = 0; s < QST; ++s) {
      mbar_init(&bars->qfull[s], 1);
      mbar_init(&bars->qempty[s], 2);   // one commit from each issuer
    }
    mbar_init(&bars->sfull, 1);
    mbar_init(&bars->dpfull, 1);
    mbar_init(&bars->pready, kSoftmax);
    mbar_init(&bars->dsready, kSoftmax);
    mbar_init(&bars->sissued[0], 1);
    mbar_init(&bars->sissued[1], 1);
    mbar_init(&bars->done, 2);
    fence_mbar_init();
  }
  if (threadIdx.x < 2 * KV_M) {                      // the constant A rows of the extra step
    const uint32_t mh = pack_bf16x2(-0.5f, -0.5f), m0 = pack_bf16x2(-0.5f, 0.f);
    *reinterpret_cast<uint4*>(smem + Lay::kaug + threadIdx.x * 16) = make_uint4(mh, m0, 0u, 0u);
    fence_async_smem();
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
    // Producer warp: lane 0 issues the TMA loads; all lanes build the B rows
    // of the extra K step for each query tile (rows lane + 32 j).
    if (lane == 0) {
      mbar_expect_tx(&bars->kvfull, 2 * KV_M * HD * 2);
      for (int blk = 0; blk < HD / 64; ++blk) {
        tma_load_3d(&tmK, &bars->kvfull, smem + Lay::k + blk * KV_M * 128, 64 * blk, kt * KV_M, bh);
        tma_load_3d(&tmV, &bars->kvfull, smem + Lay::v + blk * KV_M * 128, 64 * blk, kt * KV_M, bh);
      }
    }
    const float inv_scale = 1.f / scale;
    float ln[4], dn[4];                              // next tile's LSE / D, rows past S: 0
    auto fetch = [&](int it) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int q = (i0 + it) * Q_N + lane + 32 * j;
        ln[j] = q < S ? __ldg(lse + (int64_t)bh * S + q) * inv_scale : 0.f;
        dn[j] = q < S ? __ldg(delta + (int64_t)bh * S + q) : 0.f;
      }
    };
    // x -> (hi, mid, lo) bf16 with hi + mid + lo = x to fp32 precision, as one
    // 16-byte half row (hi, mid, lo, 0, 0, 0, 0, 0)
    auto split3 = [](float x) -> uint4 {
      const uint32_t h2 = pack_bf16x2(x, 0.f);
      const float r1 = x - __uint_as_float(h2 << 16);
      const uint32_t m2 = pack_bf16x2(r1, 0.f);
      const float r2 = r1 - __uint_as_float(m2 << 16);
      return make_uint4((h2 & 0xffffu) | (m2 << 16), pack_bf16x2(r2, 0.f), 0u, 0u);
    };
    fetch(0);
    for (int it = 0; it < n_it; ++it) {
      const int s = it % QST;
      float lc[4], dc[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) { lc[j] = ln[j]; dc[j] = dn[j]; }
      if (it + 1 < n_it) fetch(it + 1);
      if (!mbar_wait_w(&bars->qempty[s], ((it / QST) & 1) ^ 1, status, 21)) break;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = lane + 32 * j;
        const uint4 wl = split3(lc[j]), wd = split3(dc[j]);
        uint8_t* ql = smem + Lay::qaug + s * Q_N * 32 + r * 32;
        uint8_t* ol = smem + Lay::oaug + s * Q_N * 32 + r * 32;
        *reinterpret_cast<uint4*>(ql) = wl;
        *reinterpret_cast<uint4*>(ql + 16) = wl;
        *reinterpret_cast<uint4*>(ol) = wd;
        *reinterpret_cast<uint4*>(ol + 16) = wd;
      }
      fence_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_expect_tx(&bars->qfull[s], 2 * Q_N * HD * 2);
        const int row = (i0 + it) * Q_N;
        for (int blk = 0; blk < HD / 64; ++blk) {
          tma_load_3d(&tmQ, &bars->qfull[s], smem + Lay::q + s * Q_N * HD * 2 + blk * Q_N * 128,
                      64 * blk, row, bh);
          tma_load_3d(&tmO, &bars->qfull[s], smem + Lay::dO + s * Q_N * HD * 2 + blk * Q_N * 128,
                      64 * blk, row, bh);
        }
      }
      __syncwarp();
    }
  } else if (warp == 1 || warp == 10) {
    // Issuer A (warp 1): S^T = K Q^T and dV += P^T dO.  Issuer B (warp 10):
    // dP^T = V dO^T and dK += dS^T Q.  Whole-warp loops, one lane issues.
    const bool isA = warp == 1;
    constexpr uint32_t idS = idesc_bf16(KV_M, Q_N, 0, 0);   // S^T, dP^T
    constexpr uint32_t idG = idesc_bf16(KV_M, HD, 0, 1);    // dV, dK (B MN-major)
    const uint32_t sA = smem_u32(smem + (isA ? Lay::k : Lay::v));         // K or V
    const uint32_t sKaug = smem_u32(smem + Lay::kaug);
    const uint32_t sBaug = smem_u32(smem + (isA ? Lay::qaug : Lay::oaug)); // -LSE/scale or -D
    const uint32_t sB = smem_u32(smem + (isA ? Lay::q : Lay::dO));        // Q or dO ring
    const uint32_t sG = smem_u32(smem + (isA ? Lay::dO : Lay::q));        // dO or Q ring
    const uint32_t dSc = tmem + (isA ? 0u : 128u);                        // S^T or dP^T
    const uint32_t dAcc = tmem + 256 + (isA ? 0u : (uint32_t)HD);         // dV or dK
    uint64_t* ready = isA ? &bars->pready : &bars->dsready;
    uint64_t* full = isA ? &bars->sfull : &bars->dpfull;
    bool ok = mbar_wait_w(&bars->kvfull, 0, status, 22);
    for (int it = 0; ok && it <= n_it; ++it) {
      if (!isA && it < n_it &&
          !mbar_wait_w(&bars->sissued[it & 1], (it >> 1) & 1, status, 20)) { ok = false; break; }
      if (it > 0) {
        // gradient MMAs of tile it - 1: A operand = P^T / dS^T (bf16 in TMEM)
        const int sp = (it - 1) % QST;
        if (!mbar_wait_w(ready, (it - 1) & 1, status, isA ? 23 : 24)) { ok = false; break; }
        tc_fence_after();
        const uint32_t gb = sG + sp * Q_N * HD * 2;
#pragma unroll
        for (int ks = 0; ks < Q_N / 16; ++ks)
          mma_bf16_ts_w(dAcc, dSc + (ks >> 2) * 64 + (ks & 3) * 8,
                        sdesc_sw128(gb + ks * 16 * 128, Q_N * 128, 1024), idG,
                        (it > 1 || ks > 0) ? 1u : 0u);
        mma_commit_w(&bars->qempty[sp]);
      }
      if (it == n_it) break;
      const int s = it % QST;
      if (!mbar_wait_w(&bars->qfull[s], (it / QST) & 1, status, isA ? 25 : 26)) { ok = false; break; }
      tc_fence_after();
      const uint32_t bb = sB + s * Q_N * HD * 2;
#pragma unroll
      for (int ks = 0; ks < HD / 16; ++ks) {
        const uint32_t aoff = (ks >> 2) * KV_M * 128 + (ks & 3) * 32;
        const uint32_t boff = (ks >> 2) * Q_N * 128 + (ks & 3) * 32;
        mma_bf16_w(dSc, sdesc_sw128(sA + aoff, 16, 1024), sdesc_sw128(bb + boff, 16, 1024), idS,
                   ks > 0 ? 1u : 0u);
      }
      mma_bf16_w(dSc, sdesc_sw32(sKaug), sdesc_sw32(sBaug + s * Q_N * 32), idS, 1u);
      mma_commit_w(full);
      if (isA && lane == 0) mbar_arrive(&bars->sissued[it & 1]);
    }
    if (ok) mma_commit_w(&bars->done);
  } else {
    // Softmax warpgroups: warp w owns TMEM lanes 32 (w % 4) .. +31 (key rows)
    // and query columns 64 h .. 64 h + 63 of each tile, h = (w - 2) / 4.
    const int quarter = warp & 3;
    const int h = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const int kvrow = kt * KV_M + r;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const uint32_t cS = tmem + lane_addr + h * 64, cP = tmem + lane_addr + 128 + h * 64;
    const float c = scale * kLog2e;
    bool ok = true;
    for (int it = 0; ok && it < n_it; ++it) {
      const int qc0 = (i0 + it) * Q_N + h * 64;      // first query column of this thread
      const bool diag = !full && it == 0;
      // ---- P = exp2(c (s - LSE / scale)): fp32 kept in registers, bf16 into TMEM
      uint32_t p[64];                                // scores, then P (fp32 bits)
      const uint64_t c2 = f2_pack(c, c);
      if (!mbar_wait(&bars->sfull, it & 1, status, 27)) { ok = false; break; }
      tc_fence_after();
      tmem_ld32(cS, *reinterpret_cast<uint32_t(*)[32]>(&p[0]));
      tmem_ld32(cS + 32, *reinterpret_cast<uint32_t(*)[32]>(&p[32]));
      tmem_ld_wait();
      // two copies of the loop, so that off-diagonal tiles carry no
      // per-column compare
      auto p_tile = [&](auto masked) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          uint32_t pk[8];
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const int j = ch * 16 + e;
            const float2 x = f2_unpack(f2_mul(f2_pack(__uint_as_float(p[j]), __uint_as_float(p[j + 1])), c2));
            float p0 = ex2(x.x);
            float p1 = ex2(x.y);
            if constexpr (decltype(masked)::value) {
              p0 = (qc0 + j >= kvrow) ? p0 : 0.f;
              p1 = (qc0 + j + 1 >= kvrow) ? p1 : 0.f;
            }
            p[j] = __float_as_uint(p0);
            p[j + 1] = __float_as_uint(p1);
            pk[e >> 1] = pack_bf16x2(p0, p1);
          }
          // packed P of columns 16 ch .. 16 ch + 15 lands on fp32 columns
          // 8 ch .. 8 ch + 7 of this thread's range, already read above
          tmem_st8(cS + ch * 8, pk);
        }
      };
      if (diag) p_tile(std::true_type{});
      else p_tile(std::false_type{});
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->pready);
      // ---- dS = P (dP - D), bf16 into TMEM; the dP loads run one chunk ahead
      if (!mbar_wait(&bars->dpfull, it & 1, status, 28)) { ok = false; break; }
      tc_fence_after();
      uint32_t pr[2][16];
      tmem_ld16(cP, pr[0]);
      tmem_ld_wait();
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        if (ch < 3) tmem_ld16(cP + (ch + 1) * 16, pr[(ch + 1) & 1]);
        const uint32_t* q = pr[ch & 1];
        uint32_t dk[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const int j = ch * 16 + e;
          const float2 ds = f2_unpack(f2_mul(f2_pack(__uint_as_float(p[j]), __uint_as_float(p[j + 1])),
                                             f2_pack(__uint_as_float(q[e]), __uint_as_float(q[e + 1]))));
          dk[e >> 1] = pack_bf16x2(ds.x, ds.y);
        }
        // chunk ch's packed dS covers fp32 columns 8 ch .. 8 ch + 7, all
        // read by the loads of chunks <= ch, which have completed
        tmem_st8(cP + ch * 8, dk);
        if (ch < 3) tmem_ld_wait();
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(&bars->dsready);
    }
    if (ok && mbar_wait(&bars->done, 0, status, 29)) {
      tc_fence_after();
      const int which = h;                           // warpgroup 0 writes dV, 1 writes dK
      uint4* dst = (which ? dkg : dvg) + ((int64_t)bh * S + kvrow) * (HD / 8);
      const float mul = which ? scale : 1.f;
      const bool chain = !(first && last);
      float4* acc = chain ? reinterpret_cast<float4*>(which ? dk_acc : dv_acc) +
                                ((int64_t)bh * S + kvrow) * (HD / 4)
                          : nullptr;
#pragma unroll
      for (int cchunk = 0; cchunk < HD / 32; ++cchunk) {
        uint32_t o[32];
        tmem_ld32(tmem + lane_addr + 256 + which * HD + cchunk * 32, o);
        tmem_ld_wait();
        if (kvrow < S && chain) {
          lh_chain_store(o, mul, acc + cchunk * 8, dst + cchunk * 4, first, last);
        } else if (kvrow < S) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[v * 8 + 0]) * mul, __uint_as_float(o[v * 8 + 1]) * mul);
            w.y = pack_bf16x2(__uint_as_float(o[v * 8 + 2]) * mul, __uint_as_float(o[v * 8 + 3]) * mul);
            w.z = pack_bf16x2(__uint_as_float(o[v * 8 + 4]) * mul, __uint_as_float(o[v * 8 + 5]) * mul);
            w.w = pack_bf16x2(__uint_as_float(o[v * 8 + 6]) * mul, __uint_as_float(o[v * 8 + 7]) * mul);
            dst[cchunk * 4 + v] = w;
          }
        }
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

// --------------------------------------------------------------------- dQ --

constexpr int Q_M = 128;   // stationary query rows
constexpr int KV_N = 128;  // walked key rows per tile
constexpr int KST = 3;     // stages of the walked K ring (K is held until the dQ MMAs)
constexpr int VST = 2;     // stages of the walked V ring (V only until the dP MMAs)
// dS goes back to the dQ MMAs in kDsGroups groups of key columns per
// warpgroup, each on its own barrier, so the dQ MMAs of a group run while the
// softmax still works on the next.
constexpr int kDsGroups = 2;

// warp 0 TMA, warp 1 issuer A (S), warps 2-9 softmax, warp 10 issuer B (dQ, dP)
constexpr int kThreadsDq = 352;

template <int HD>
struct DqLayout {
  static constexpr uint32_t q = 0;
  static constexpr uint32_t dO = q + Q_M * HD * 2;
  static constexpr uint32_t k = dO + Q_M * HD * 2;          // KST stages
  static constexpr uint32_t v = k + KST * KV_N * HD * 2;     // VST stages
  static constexpr uint32_t bar = v + VST * KV_N * HD * 2;
  static constexpr uint32_t bytes = bar + 256;
};

struct DqBars {
  // dpissued[t % 2]: issuer B has issued dP(t).  Issuer A waits for it before
  // S(t + 1), so B's MMAs (dQ, dP: the softmax's critical chain) enter the
  // tensor pipe first and A's fill the time B waits for the softmax.  Two
  // barriers by parity, because B may run one step ahead of A's wait.
  uint64_t qfull, kfull[KST], kempty[KST], vfull[VST], vempty[VST], sfull[2], sfree[2], dpfull,
      dsready[kDsGroups], dpissued[2], done;
  uint32_t tmem_base;
};

// TMEM columns: S buffers 0 / 128, dP 256..383 (dS as packed bf16 over the
// first 32 columns of each warpgroup's 64), dQ 384.
//
// Issuer A computes S(j) = Q K(j)^T into the S buffer j % 2 as soon as the
// softmax has read S(j - 2); issuer B runs dQ += dS(j - 1) K(j - 1) (group
// by group, as the softmax hands dS back in kDsGroups groups of keys), then
// dP(j) = dO V(j)^T (in issue order, so dP(j) overwrites dS(j - 1) only
// after the dQ MMAs that read it).  The softmax turns S(j) into P in
// registers while B's MMAs run, then dP(j) into dS.  LSE and D are
// per-row values, so the softmax threads (one query row each) hold them in
// registers and read nothing but TMEM in the loop.
template <int HD>
__global__ void __launch_bounds__(kThreadsDq, 1)
    k_attn_bwd_dq(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
                  const __grid_constant__ CUtensorMap tmV, const __grid_constant__ CUtensorMap tmO,
                  const float* __restrict__ lse, const float* __restrict__ delta,
                  uint4* __restrict__ dqg, int S, int BH, float scale, int* status, int full,
                  int first, int last, float* __restrict__ dq_acc) {
  using Lay = DqLayout<HD>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~(uintptr_t)1023);
  DqBars* bars = reinterpret_cast<DqBars*>(smem + Lay::bar);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_qt = (S + Q_M - 1) / Q_M;
  const int qt = n_qt - 1 - (int)(blockIdx.x / BH);  // longest rows first
  const int bh = (int)(blockIdx.x % BH);
  const int n_kv = full ? n_qt : qt + 1;             // key tiles up to the diagonal (KV_N == Q_M)

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
    for (int s = 0; s < 2; ++s) {
      mbar_init(&bars->sfull[s], 1);
      mbar_init(&bars->sfree[s], kSoftmax);
    }
    mbar_init(&bars->dpfull, 1);
    for (int g = 0; g < kDsGroups; ++g) mbar_init(&bars->dsready[g], kSoftmax);
    mbar_init(&bars->dpissued[0], 1);
    mbar_init(&bars->dpissued[1], 1);
    mbar_init(&bars->done, 1);
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
      mbar_expect_tx(&bars->qfull, 2 * Q_M * HD * 2);
      for (int blk = 0; blk < HD / 64; ++blk) {
        tma_load_3d(&tmQ, &bars->qfull, smem + Lay::q + blk * Q_M * 128, 64 * blk, qt * Q_M, bh);
        tma_load_3d(&tmO, &bars->qfull, smem + Lay::dO + blk * Q_M * 128, 64 * blk, qt * Q_M, bh);
      }
      for (int j = 0; j < n_kv; ++j) {
        const int s = j % KST, t = j % VST;
        if (!mbar_wait(&bars->kempty[s], ((j / KST) & 1) ^ 1, status, 31)) break;
        mbar_expect_tx(&bars->kfull[s], KV_N * HD * 2);
        for (int blk = 0; blk < HD / 64; ++blk)
          tma_load_3d(&tmK, &bars->kfull[s], smem + Lay::k + s * KV_N * HD * 2 + blk * KV_N * 128,
                      64 * blk, j * KV_N, bh);
        if (!mbar_wait(&bars->vempty[t], ((j / VST) & 1) ^ 1, status, 30)) break;
        mbar_expect_tx(&bars->vfull[t], KV_N * HD * 2);
        for (int blk = 0; blk < HD / 64; ++blk)
          tma_load_3d(&tmV, &bars->vfull[t], smem + Lay::v + t * KV_N * HD * 2 + blk * KV_N * 128,
                      64 * blk, j * KV_N, bh);
      }
    }
  } else if (warp == 1) {
    // Issuer A: S(j) = Q K(j)^T into buffer j % 2.  Whole-warp loop.
    constexpr uint32_t idS = idesc_bf16(Q_M, KV_N, 0, 0);
    const uint32_t sQ = smem_u32(smem + Lay::q), sK = smem_u32(smem + Lay::k);
    bool ok = mbar_wait_w(&bars->qfull, 0, status, 32);
    for (int j = 0; ok && j < n_kv; ++j) {
      const int s = j % KST, sb = j & 1;
      if (!mbar_wait_w(&bars->kfull[s], (j / KST) & 1, status, 33)) break;
      if (!mbar_wait_w(&bars->sfree[sb], ((j >> 1) & 1) ^ 1, status, 34)) break;
      if (j > 0 && !mbar_wait_w(&bars->dpissued[(j - 1) & 1], ((j - 1) >> 1) & 1, status, 29)) break;
      tc_fence_after();
      const uint32_t kb = sK + s * KV_N * HD * 2;
#pragma unroll
      for (int ks = 0; ks < HD / 16; ++ks) {
        const uint32_t qoff = (ks >> 2) * Q_M * 128 + (ks & 3) * 32;
        const uint32_t koff = (ks >> 2) * KV_N * 128 + (ks & 3) * 32;
        mma_bf16_w(tmem + sb * KV_N, sdesc_sw128(sQ + qoff, 16, 1024),
                   sdesc_sw128(kb + koff, 16, 1024), idS, ks > 0 ? 1u : 0u);
      }
      mma_commit_w(&bars->sfull[sb]);
    }
  } else if (warp == 10) {
    // Issuer B: dQ += dS(j - 1) K(j - 1) (A operand from TMEM), then
    // dP(j) = dO V(j)^T.  Whole-warp loop.
    constexpr uint32_t idS = idesc_bf16(Q_M, KV_N, 0, 0);
    constexpr uint32_t idG = idesc_bf16(Q_M, HD, 0, 1);     // dQ (B = K, MN-major)
    const uint32_t sO = smem_u32(smem + Lay::dO), sK = smem_u32(smem + Lay::k);
    const uint32_t sV = smem_u32(smem + Lay::v);
    bool ok = mbar_wait_w(&bars->qfull, 0, status, 35);
    for (int j = 0; ok && j <= n_kv; ++j) {
      if (j > 0) {
        // group by group as the softmax hands dS back: group g is key steps
        // ks = 4 h + c of both warpgroups h, c in [g, g + 1) * 4 / kDsGroups
        const int sp = (j - 1) % KST;
        const uint32_t kb = sK + sp * KV_N * HD * 2;
#pragma unroll
        for (int g = 0; g < kDsGroups; ++g) {
          if (!mbar_wait_w(&bars->dsready[g], (j - 1) & 1, status, 36)) { ok = false; break; }
          tc_fence_after();
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
#pragma unroll
            for (int c = g * (4 / kDsGroups); c < (g + 1) * (4 / kDsGroups); ++c) {
              const int ks = 4 * hh + c;
              mma_bf16_ts_w(tmem + 384, tmem + 256 + hh * 64 + c * 8,
                            sdesc_sw128(kb + ks * 16 * 128, KV_N * 128, 1024), idG,
                            (j > 1 || ks > 0) ? 1u : 0u);
            }
        }
        if (!ok) break;
        mma_commit_w(&bars->kempty[sp]);
      }
      if (j == n_kv) break;
      const int t = j % VST;
      if (!mbar_wait_w(&bars->vfull[t], (j / VST) & 1, status, 37)) { ok = false; break; }
      tc_fence_after();
      const uint32_t vb = sV + t * KV_N * HD * 2;
#pragma unroll
      for (int ks = 0; ks < HD / 16; ++ks) {
        const uint32_t qoff = (ks >> 2) * Q_M * 128 + (ks & 3) * 32;
        const uint32_t koff = (ks >> 2) * KV_N * 128 + (ks & 3) * 32;
        mma_bf16_w(tmem + 256, sdesc_sw128(sO + qoff, 16, 1024), sdesc_sw128(vb + koff, 16, 1024),
                   idS, ks > 0 ? 1u : 0u);
      }
      mma_commit_w(&bars->dpfull);
      mma_commit_w(&bars->vempty[t]);
      if (lane == 0) mbar_arrive(&bars->dpissued[j & 1]);
    }
    if (ok) mma_commit_w(&bars->done);
  } else {
    // Softmax warpgroups: warp w owns TMEM lanes 32 (w % 4) .. +31 (query
    // rows) and key columns 64 h .. 64 h + 63 of each tile, h = (w - 2) / 4.
    const int quarter = warp & 3;
    const int h = (warp - 2) >> 2;
    const int r = quarter * 32 + lane;
    const int qrow = qt * Q_M + r;
    const uint32_t lane_addr = (uint32_t)(quarter * 32) << 16;
    const uint32_t cP = tmem + lane_addr + 256 + h * 64;
    const float c = scale * kLog2e;
    const float lrow = qrow < S ? __ldg(lse + (int64_t)bh * S + qrow) * kLog2e : INFINITY;
    const float drow = qrow < S ? __ldg(delta + (int64_t)bh * S + qrow) : 0.f;
    bool ok = true;
    for (int j = 0; ok && j < n_kv; ++j) {
      const int sb = j & 1;
      const int kc0 = j * KV_N + h * 64;               // first key column of this thread
      const bool diag = !full && j == qt;
      // ---- P = exp2(c s - lse), fp32 in registers
      uint32_t p[64];
      if (!mbar_wait(&bars->sfull[sb], (j >> 1) & 1, status, 38)) { ok = false; break; }
      tc_fence_after();
      const uint32_t cS = tmem + lane_addr + sb * KV_N + h * 64;
      tmem_ld32(cS, *reinterpret_cast<uint32_t(*)[32]>(&p[0]));
      tmem_ld32(cS + 32, *reinterpret_cast<uint32_t(*)[32]>(&p[32]));
      tmem_ld_wait();
      tc_fence_before();
      mbar_arrive(&bars->sfree[sb]);
      const uint64_t c2 = f2_pack(c, c), nl2 = f2_pack(-lrow, -lrow);
      auto p_row = [&](auto masked) {   // two copies: no compare off the diagonal
#pragma unroll
        for (int e = 0; e < 64; e += 2) {
          const float2 x = f2_unpack(f2_fma(f2_pack(__uint_as_float(p[e]), __uint_as_float(p[e + 1])), c2, nl2));
          float p0 = ex2(x.x), p1 = ex2(x.y);
          if constexpr (decltype(masked)::value) {
            p0 = (kc0 + e <= qrow) ? p0 : 0.f;
            p1 = (kc0 + e + 1 <= qrow) ? p1 : 0.f;
          }
          p[e] = __float_as_uint(p0);
          p[e + 1] = __float_as_uint(p1);
        }
      };
      if (diag) p_row(std::true_type{});
      else p_row(std::false_type{});
#pragma unroll
      for (int g = 0; g < 4; ++g) materialize16(p + 16 * g);
      // ---- dS = P (dP - D), bf16 into TMEM; the dP loads run one chunk ahead
      if (!mbar_wait(&bars->dpfull, j & 1, status, 39)) { ok = false; break; }
      tc_fence_after();
      const uint64_t nd2 = f2_pack(-drow, -drow);
      uint32_t pr[2][16];
      tmem_ld16(cP, pr[0]);
      tmem_ld_wait();
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        if (ch < 3) tmem_ld16(cP + (ch + 1) * 16, pr[(ch + 1) & 1]);
        const uint32_t* q = pr[ch & 1];
        uint32_t dk[8];
#pragma unroll
        for (int e = 0; e < 16; e += 2) {
          const int i = ch * 16 + e;
          const float2 ds = f2_unpack(f2_mul(f2_pack(__uint_as_float(p[i]), __uint_as_float(p[i + 1])),
                                             f2_add(f2_pack(__uint_as_float(q[e]), __uint_as_float(q[e + 1])), nd2)));
          dk[e >> 1] = pack_bf16x2(ds.x, ds.y);
        }
        // chunk ch's packed dS covers fp32 columns 8 ch .. 8 ch + 7, all
        // read by the loads of chunks <= ch, which have completed
        tmem_st8(cP + ch * 8, dk);
        if ((ch + 1) % (4 / kDsGroups) == 0) {       // group complete: hand it back
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(&bars->dsready[ch / (4 / kDsGroups)]);
        }
        if (ch < 3) tmem_ld_wait();
      }
    }
    if (ok && mbar_wait(&bars->done, 0, status, 40)) {
      tc_fence_after();
      uint4* dst = dqg + ((int64_t)bh * S + qrow) * (HD / 8);
      const bool chain = !(first && last);
      float4* acc = chain ? reinterpret_cast<float4*>(dq_acc) + ((int64_t)bh * S + qrow) * (HD / 4)
                          : nullptr;
#pragma unroll
      for (int q = 0; q < HD / 64; ++q) {            // each warpgroup: half of the d columns
        const int cchunk = h * (HD / 64) + q;
        uint32_t o[32];
        tmem_ld32(tmem + lane_addr + 384 + cchunk * 32, o);
        tmem_ld_wait();
        if (qrow < S && chain) {
          lh_chain_store(o, scale, acc + cchunk * 8, dst + cchunk * 4, first, last);
        } else if (qrow < S) {
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            uint4 w;
            w.x = pack_bf16x2(__uint_as_float(o[v * 8 + 0]) * scale, __uint_as_float(o[v * 8 + 1]) * scale);
            w.y = pack_bf16x2(__uint_as_float(o[v * 8 + 2]) * scale, __uint_as_float(o[v * 8 + 3]) * scale);
            w.z = pack_bf16x2(__uint_as_float(o[v * 8 + 4]) * scale, __uint_as_float(o[v * 8 + 5]) * scale);
            w.w = pack_bf16x2(__uint_as_float(o[v * 8 + 6]) * scale, __uint_as_float(o[v * 8 + 7]) * scale);
            dst[cchunk * 4 + v] = w;
          }
        }
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

// Both kernels take one CTA per SM (they allocate 512 TMEM columns).
constexpr uint32_t kSmemDkdv = DkdvLayout<128>::bytes + 1024;
constexpr uint32_t kSmemDq = DqLayout<128>::bytes + 1024;
static_assert(kSmemDkdv <= 232448 && kSmemDq <= 232448, "shared memory");
static_assert(kSmemDkdv > 232448 / 2 && kSmemDq > 232448 / 2, "one CTA per SM");

template <int HD>
cudaError_t launch_hd(int BH, int S, float scale, const CUtensorMap* maps, const float* lse,
                      const float* delta, lh_bf16* dqg, lh_bf16* dkg, lh_bf16* dvg, int* status,
                      cudaStream_t st, int which, const LhRingStep& rs) {
  // maps: Q, K, V, dO with 128-row boxes (every tile of both kernels)
  if (which & 1) {
    cudaFuncSetAttribute(k_attn_bwd_dkdv<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemDkdv);
    const int n_kt = (S + KV_M - 1) / KV_M;
    k_attn_bwd_dkdv<HD><<<n_kt * BH, kThreadsDkdv, kSmemDkdv, st>>>(
        maps[0], maps[1], maps[2], maps[3], lse, delta, (uint4*)dkg, (uint4*)dvg, S, BH, scale,
        status, rs.full, rs.kv_first, rs.kv_last, rs.dk_acc, rs.dv_acc);
  }
  if (which & 2) {
    cudaFuncSetAttribute(k_attn_bwd_dq<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemDq);
    const int n_qt = (S + Q_M - 1) / Q_M;
    k_attn_bwd_dq<HD><<<n_qt * BH, kThreadsDq, kSmemDq, st>>>(maps[0], maps[1], maps[2], maps[3],
                                                             lse, delta, (uint4*)dqg, S, BH, scale,
                                                             status, rs.full, rs.q_first,
                                                             rs.q_last, rs.dq_acc);
  }
  return cudaGetLastError();
}

}  // namespace

bool lh_make_tmap_3d(CUtensorMap* m, const void* base, int64_t BH, int64_t rows, int d,
                     int box_rows);

cudaError_t lh_launch_attn_bwd(int BH, int64_t S, int d, float scale, const lh_bf16* qg,
                               const lh_bf16* kg, const lh_bf16* vg, const lh_bf16* dog,
                               const float* lse, const float* delta, lh_bf16* dqg,
                               lh_bf16* dkg, lh_bf16* dvg, int* status, cudaStream_t st,
                               int which, const LhRingStep* ring) {
  const LhRingStep plain{};
  const LhRingStep& rs = ring ? *ring : plain;
  CUtensorMap maps[4];
  const lh_bf16* src[4] = {qg, kg, vg, dog};
  for (int i = 0; i < 4; ++i)
    if (!lh_make_tmap_3d(&maps[i], src[i], BH, S, d, 128)) return cudaErrorInvalidValue;
  if (d == 128)
    return launch_hd<128>(BH, (int)S, scale, maps, lse, delta, dqg, dkg, dvg, status, st, which, rs);
  if (d == 64)
    return launch_hd<64>(BH, (int)S, scale, maps, lse, delta, dqg, dkg, dvg, status, st, which, rs);
  return cudaErrorInvalidValue;
}
