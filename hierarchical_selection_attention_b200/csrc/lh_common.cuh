// Internal helpers shared by the Lighthouse kernels: derived sizes, bf16
// packing, the device status word and bounded waits.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lighthouse.h"

#define LH_MAX_LEVELS 8

// Sizes derived once on the host from an lh_config and passed by value.
struct LhDims {
  int B, H, d, L, p;
  int64_t N;
  int64_t S;                      // gathered length (Eq. 8)
  int64_t P;                      // pyramid entries per (b, h)
  int64_t n_cand;                 // entries of levels 0..L-2
  int64_t n_sel;                  // (L-1) p k
  int64_t lvl_size[LH_MAX_LEVELS];   // N / p^l
  int64_t lvl_off[LH_MAX_LEVELS];    // flat offset of level l
  int64_t lvl_span[LH_MAX_LEVELS];   // p^l
  int64_t pool_row[LH_MAX_LEVELS];   // first pooled row of level l (l >= 1), per batch row
  int64_t pooled_rows;               // sum_{l>=1} N / p^l
  // Selection segments: select_mode 0 has one (all finer entries, n_sel to
  // take), select_mode 1 one per finer level (p k to take from each),
  // select_mode 2 one per chunk (nseg chunks of the n_cand candidates, chunk
  // s = [floor(s n_cand / nseg), floor((s+1) n_cand / nseg)), seg_need each;
  // seg_lo / seg_len are not used).
  int select_mode;
  int nseg;
  int64_t seg_lo[LH_MAX_LEVELS];     // first flat index of segment s
  int64_t seg_len[LH_MAX_LEVELS];    // its entries
  int64_t seg_need;                  // entries to take from each segment
  float scale;
  int* status;                       // device status word [code, detail]
};

// Device status word: first error wins.  Codes are lh_status values; the
// detail word says which wait or check failed.
__device__ __forceinline__ void lh_report(int* status, int code, int detail) {
  if (atomicCAS(status, 0, code) == 0) atomicExch(status + 1, detail);
}

// Level of a flat pyramid index (levels are few; a linear scan is cheapest).
__device__ __forceinline__ int lh_level_of(const LhDims& D, int64_t f) {
  int l = 0;
#pragma unroll 1
  for (int j = 1; j < D.L; ++j)
    if (f >= D.lvl_off[j]) l = j;
  return l;
}

// 16-byte asynchronous copy global -> shared (cp.async, L1 bypassed), its
// commit group and the wait for all but the N most recent groups.  Used where
// a thread copies into shared-memory slots that only it reads back, so the
// wait alone orders the copy before the read.
__device__ __forceinline__ void lh_cp_async16(uint4* dst, const uint4* src) {
  const uint32_t d = (uint32_t)__cvta_generic_to_shared(dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(src) : "memory");
}

__device__ __forceinline__ void lh_cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}

template <int N>
__device__ __forceinline__ void lh_cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float2 unpack_bf16x2(uint32_t u) {
  float2 r;
  r.x = __uint_as_float(u << 16);
  r.y = __uint_as_float(u & 0xffff0000u);
  return r;
}

// Host side launchers (one per kernel family), all enqueue on `st`.
cudaError_t lh_launch_pyramid(const LhDims& D, const lh_bf16* q, const lh_bf16* k,
                              const lh_bf16* v, lh_bf16* q_lv, lh_bf16* k_lv, lh_bf16* v_lv,
                              float* qk, float* kq, cudaStream_t st);
size_t lh_select_ws_bytes(const LhDims& D);
cudaError_t lh_launch_select(const LhDims& D, const float* qk, const float* kq,
                             int32_t* sel_idx, int32_t* slot_map, void* ws, cudaStream_t st,
                             int* launches);
cudaError_t lh_launch_gather(const LhDims& D, const lh_bf16* q, const lh_bf16* k,
                             const lh_bf16* v, const lh_bf16* q_lv, const lh_bf16* k_lv,
                             const lh_bf16* v_lv, const int32_t* sel_idx, lh_bf16* qg,
                             lh_bf16* kg, lh_bf16* vg, cudaStream_t st);
cudaError_t lh_launch_scatter(const LhDims& D, const lh_bf16* og, const int32_t* slot_map,
                              lh_bf16* o, cudaStream_t st);
size_t lh_scatter_atomic_ws_bytes(const LhDims& D);
cudaError_t lh_launch_scatter_atomic(const LhDims& D, const lh_bf16* og,
                                     const int32_t* slot_map, lh_bf16* o, void* ws,
                                     cudaStream_t st, int* launches);
cudaError_t lh_launch_scatter_bwd(const LhDims& D, const lh_bf16* dout, const lh_bf16* og,
                                  const lh_bf16* og_lo, const int32_t* sel_idx, lh_bf16* dog,
                                  float* delta, cudaStream_t st);
cudaError_t lh_launch_gather_bwd(const LhDims& D, const lh_bf16* dqg, const lh_bf16* dkg,
                                 const lh_bf16* dvg, const int32_t* slot_map, lh_bf16* dq,
                                 lh_bf16* dk, lh_bf16* dv, cudaStream_t st);
// full: the K/V block is an earlier shard's (every key visible); first /
// last: see the ring-step merge in lh_attn_fwd.cu.  The plain layer passes
// full = 0, first = last = 1 and no accumulators.
cudaError_t lh_launch_attn_fwd(int BH, int64_t S, int d, float scale, const lh_bf16* qg,
                               const lh_bf16* kg, const lh_bf16* vg, lh_bf16* og,
                               lh_bf16* og_lo, float* lse, int* status, cudaStream_t st,
                               int full = 0, int first = 1, int last = 1,
                               float* o_acc = nullptr, float* lse2_acc = nullptr);
// One ring step of the attention backward: the mode, and for each side (the
// query rows' dQ; the key block's dK, dV) whether this step opens or closes
// its fp32 sum.  Zero-initialised it is the plain single-block backward.
struct LhRingStep {
  int full = 0;
  int q_first = 1, q_last = 1, kv_first = 1, kv_last = 1;
  float* dq_acc = nullptr;
  float* dk_acc = nullptr;
  float* dv_acc = nullptr;
};
cudaError_t lh_launch_attn_delta(int BH, int64_t S, int d, const lh_bf16* og,
                                 const lh_bf16* og_lo, const lh_bf16* dog, float* delta,
                                 cudaStream_t st);
// which: 1 = dK/dV kernel, 2 = dQ kernel, 3 = both.
cudaError_t lh_launch_attn_bwd(int BH, int64_t S, int d, float scale, const lh_bf16* qg,
                               const lh_bf16* kg, const lh_bf16* vg, const lh_bf16* dog,
                               const float* lse, const float* delta, lh_bf16* dqg,
                               lh_bf16* dkg, lh_bf16* dvg, int* status, cudaStream_t st,
                               int which, const LhRingStep* ring = nullptr);

// One warp waiting on an mbarrier nothing completes (lh_selftest.cu).
cudaError_t lh_launch_wait_timeout_check(int* status, int where, cudaStream_t st);

// Plain GEMM (lh_gemm.cu).
size_t lh_gemm_partial_bytes(int64_t M, int64_t N, int splits);
cudaError_t lh_launch_gemm(int64_t M, int64_t N, int npairs, const lh_gemm_operand* ops, int a_mn,
                           int b_mn, lh_bf16* c, int64_t ldc, int splits, void* ws, int* status,
                           int num_sms, cudaStream_t st, int* launches);

