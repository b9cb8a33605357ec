// C ABI of the Lighthouse Attention hot path (declared in lighthouse.h):
// argument checking, buffer layouts and the order of the launches.  No
// arithmetic of the method lives here.
#include <math.h>
#include <string.h>

#include "lh_common.cuh"

namespace {

__device__ int g_status_word[2];  // [code, detail], see lh_get_device_status

constexpr size_t kAlign = 256;
inline size_t up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

// Device address of the status word on the current device and context.
// Looked up on every call, not cached: the lookup is a table read in the
// runtime, is thread-safe, and stays right after a device reset or a new
// primary context, where a cached address would point at freed memory.
int* status_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
  return static_cast<int*>(p);
}

lh_status check(const lh_config* c) {
  if (!c) return LH_ERR_INVALID_ARGUMENT;
  if (c->B < 1 || c->N < 1 || c->H < 1 || c->p < 2 || c->L < 1 || c->k < 0)
    return LH_ERR_INVALID_ARGUMENT;
  if (c->L > 6) return LH_ERR_UNSUPPORTED;
  if (c->N >= (1LL << 31) || c->H >= (1 << 16) || c->B >= (1 << 16)) return LH_ERR_UNSUPPORTED;
  int64_t w = 1;
  for (int l = 1; l < c->L; ++l) {
    if (w > c->N / c->p) return LH_ERR_INVALID_ARGUMENT;  // p^(L-1) > N
    w *= c->p;
  }
  if (c->N % w) return LH_ERR_INVALID_ARGUMENT;  // Sec. 3.3: p^(L-1) | N
  int64_t cand = 0, P = 0, span = 1;
  for (int l = 0; l < c->L; ++l) {
    P += c->N / span;
    if (l < c->L - 1) cand += c->N / span;
    span *= (l < c->L - 1) ? c->p : 1;
  }
  if (c->k > (1LL << 31)) return LH_ERR_INVALID_ARGUMENT;
  const int64_t n_sel = (c->L - 1) * c->p * c->k;
  if (n_sel > cand) return LH_ERR_INVALID_ARGUMENT;
  if (c->select_mode == 1 && c->L > 1) {   // p k must fit in the coarsest finer level
    int64_t coarsest_finer = c->N;
    for (int l = 0; l < c->L - 2; ++l) coarsest_finer /= c->p;
    if ((int64_t)c->p * c->k > coarsest_finer) return LH_ERR_INVALID_ARGUMENT;
  }
  if (P >= (1LL << 31)) return LH_ERR_UNSUPPORTED;
  if (c->d != 64 && c->d != 128) return LH_ERR_UNSUPPORTED;
  if (c->scatter_mode != 0 && c->scatter_mode != 1) return LH_ERR_INVALID_ARGUMENT;
  if (c->select_mode < 0 || c->select_mode > 2) return LH_ERR_UNSUPPORTED;
  if (c->select_mode == 2 && n_sel > 0) {  // stratified: n_sel / m chunks of the candidates
    if (c->select_chunk < 1 || n_sel % c->select_chunk) return LH_ERR_INVALID_ARGUMENT;
    if ((int64_t)c->B * c->H * (n_sel / c->select_chunk) >= (1LL << 31)) return LH_ERR_UNSUPPORTED;
  }
  if (!(c->scale == c->scale)) return LH_ERR_INVALID_ARGUMENT;
  const int64_t S = c->N / w + n_sel;
  if (S >= (1LL << 31) || (int64_t)c->B * c->H * ((S + 127) / 128) >= (1LL << 31))
    return LH_ERR_UNSUPPORTED;
  // grids with (b, h) or (b, h) x selection segment in gridDim.y (<= 65535)
  const int64_t BH = (int64_t)c->B * c->H;
  const int64_t segs = (c->select_mode == 1 && c->L > 1) ? c->L - 1 : 1;
  if (BH * segs > 65535) return LH_ERR_UNSUPPORTED;
  return LH_OK;
}

LhDims dims(const lh_config* c) {
  LhDims D;
  memset(&D, 0, sizeof(D));
  D.B = (int)c->B; D.H = (int)c->H; D.d = (int)c->d; D.L = (int)c->L; D.p = (int)c->p;
  D.N = c->N;
  int64_t span = 1, off = 0, prow = 0;
  for (int l = 0; l < D.L; ++l) {
    D.lvl_span[l] = span;
    D.lvl_size[l] = c->N / span;
    D.lvl_off[l] = off;
    D.pool_row[l] = l == 0 ? 0 : prow;
    if (l >= 1) prow += D.lvl_size[l];
    off += D.lvl_size[l];
    span *= c->p;
  }
  D.P = off;
  D.pooled_rows = prow;
  D.n_cand = D.L > 1 ? D.lvl_off[D.L - 1] : 0;
  D.n_sel = (int64_t)(D.L - 1) * c->p * c->k;
  D.S = D.lvl_size[D.L - 1] + D.n_sel;
  D.select_mode = c->select_mode;
  if (c->select_mode == 2 && D.n_sel > 0) {
    // one segment per chunk; the chunk bounds are computed, not stored
    D.nseg = (int)(D.n_sel / c->select_chunk);
    D.seg_need = c->select_chunk;
  } else if (c->select_mode == 1 && D.L > 1) {
    D.nseg = D.L - 1;
    for (int l = 0; l < D.L - 1; ++l) {
      D.seg_lo[l] = D.lvl_off[l];
      D.seg_len[l] = D.lvl_size[l];
    }
    D.seg_need = (int64_t)c->p * c->k;
  } else {
    D.select_mode = c->select_mode == 1 ? 1 : 0;   // nothing to stratify: one empty segment
    D.nseg = 1;
    D.seg_lo[0] = 0;
    D.seg_len[0] = D.n_cand;
    D.seg_need = D.n_sel;
  }
  D.scale = c->scale > 0.f ? c->scale : (float)(1.0 / sqrt((double)c->d));
  D.status = nullptr;
  return D;
}

// Dims for a call that launches kernels: adds the device status word.
LhDims launch_dims(const lh_config* c) {
  LhDims D = dims(c);
  D.status = status_ptr();
  return D;
}

struct FwdWs {
  size_t select, q_lv, k_lv, v_lv, qk, kq, atomic, total;
};

FwdWs fwd_layout(const LhDims& D, int scatter_mode) {
  FwdWs w;
  const size_t pooled = (size_t)D.B * D.pooled_rows * D.H * D.d * 2;
  const size_t sc = (size_t)D.B * D.H * D.P * 4;
  size_t o = 0;
  w.select = o; o += up(lh_select_ws_bytes(D));
  w.q_lv = o; o += up(pooled);
  w.k_lv = o; o += up(pooled);
  w.v_lv = o; o += up(pooled);
  w.qk = o; o += up(sc);
  w.kq = o; o += up(sc);
  w.atomic = o; o += scatter_mode == 1 ? up(lh_scatter_atomic_ws_bytes(D)) : 0;
  w.total = o;
  return w;
}

constexpr int kSaved = 8;  // sel_idx, slot_map, qg, kg, vg, og, og_lo, lse

struct Saved {
  size_t off[kSaved];
  size_t total;
};

Saved saved_layout(const LhDims& D) {
  Saved s;
  const size_t rows = (size_t)D.B * D.H * D.S;
  const size_t g = rows * D.d * 2;
  const size_t sizes[kSaved] = {rows * 4, (size_t)D.B * D.H * D.P * 4, g, g, g, g, g, rows * 4};
  size_t o = 0;
  for (int i = 0; i < kSaved; ++i) {
    s.off[i] = o;
    o += up(sizes[i]);
  }
  s.total = o;
  return s;
}

struct BwdWs {
  size_t dog, delta, dqg, dkg, dvg, total;
};

BwdWs bwd_layout(const LhDims& D) {
  BwdWs b;
  const size_t rows = (size_t)D.B * D.H * D.S;
  size_t o = 0;
  b.delta = o; o += up(rows * 4);
  b.dog = o; o += up(rows * D.d * 2);
  b.dqg = o; o += up(rows * D.d * 2);
  b.dkg = o; o += up(rows * D.d * 2);
  b.dvg = o; o += up(rows * D.d * 2);
  b.total = o;
  return b;
}

inline bool aligned(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

template <typename... Ts>
inline bool all_aligned(Ts... ps) {
  bool ok = true;
  ((ok = ok && ps != nullptr && aligned(ps)), ...);
  return ok;
}

inline lh_status cu(cudaError_t e) { return e == cudaSuccess ? LH_OK : LH_ERR_CUDA; }

template <typename T>
inline T* at(void* base, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(base) + off);
}
template <typename T>
inline const T* at(const void* base, size_t off) {
  return reinterpret_cast<const T*>(static_cast<const char*>(base) + off);
}

#define LH_TRY(expr)                   \
  do {                                 \
    lh_status _s = (expr);             \
    if (_s != LH_OK) return _s;        \
  } while (0)

}  // namespace

extern "C" {

lh_status lh_config_check(const lh_config* cfg) { return check(cfg); }

int64_t lh_subseq_len(const lh_config* cfg) {
  if (check(cfg) != LH_OK) return -1;
  return dims(cfg).S;
}

int64_t lh_total_entries(const lh_config* cfg) {
  if (check(cfg) != LH_OK) return -1;
  return dims(cfg).P;
}

int64_t lh_pooled_rows(const lh_config* cfg) {
  if (check(cfg) != LH_OK) return -1;
  return dims(cfg).pooled_rows;
}

lh_status lh_workspace_bytes(const lh_config* cfg, size_t* fwd_ws, size_t* bwd_ws,
                             size_t* saved) {
  LH_TRY(check(cfg));
  const LhDims D = dims(cfg);
  if (fwd_ws) *fwd_ws = fwd_layout(D, cfg->scatter_mode).total;
  if (bwd_ws) *bwd_ws = bwd_layout(D).total;
  if (saved) *saved = saved_layout(D).total;
  return LH_OK;
}

lh_status lh_saved_offsets(const lh_config* cfg, size_t* offsets) {
  LH_TRY(check(cfg));
  if (!offsets) return LH_ERR_INVALID_ARGUMENT;
  const Saved s = saved_layout(dims(cfg));
  for (int i = 0; i < kSaved; ++i) offsets[i] = s.off[i];
  return LH_OK;
}

lh_status lh_bwd_ws_offsets(const lh_config* cfg, size_t* offsets) {
  LH_TRY(check(cfg));
  if (!offsets) return LH_ERR_INVALID_ARGUMENT;
  const BwdWs b = bwd_layout(dims(cfg));
  offsets[0] = b.delta;
  offsets[1] = b.dog;
  offsets[2] = b.dqg;
  offsets[3] = b.dkg;
  offsets[4] = b.dvg;
  return LH_OK;
}

lh_status lh_pyramid(const lh_config* cfg, const lh_bf16* q, const lh_bf16* k,
                     const lh_bf16* v, lh_bf16* q_lv, lh_bf16* k_lv, lh_bf16* v_lv,
                     float* qk, float* kq, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(q, k, v, qk, kq)) return LH_ERR_INVALID_ARGUMENT;
  if (cfg->L > 1 && !all_aligned(q_lv, k_lv, v_lv)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  return cu(lh_launch_pyramid(D, q, k, v, q_lv, k_lv, v_lv, qk, kq, (cudaStream_t)stream));
}

lh_status lh_score_topk(const lh_config* cfg, const float* qk, const float* kq,
                        int32_t* sel_idx, int32_t* slot_map, void* ws, size_t ws_bytes,
                        void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(qk, kq, sel_idx, slot_map, ws)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  if (ws_bytes < lh_select_ws_bytes(D)) return LH_ERR_WORKSPACE;
  return cu(lh_launch_select(D, qk, kq, sel_idx, slot_map, ws, (cudaStream_t)stream, nullptr));
}

lh_status lh_gather(const lh_config* cfg, const lh_bf16* q, const lh_bf16* k,
                    const lh_bf16* v, const lh_bf16* q_lv, const lh_bf16* k_lv,
                    const lh_bf16* v_lv, const int32_t* sel_idx, lh_bf16* qg, lh_bf16* kg,
                    lh_bf16* vg, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(q, k, v, sel_idx, qg, kg, vg)) return LH_ERR_INVALID_ARGUMENT;
  if (cfg->L > 1 && !all_aligned(q_lv, k_lv, v_lv)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  return cu(lh_launch_gather(D, q, k, v, q_lv, k_lv, v_lv, sel_idx, qg, kg, vg,
                             (cudaStream_t)stream));
}

lh_status lh_attn_fwd(const lh_config* cfg, const lh_bf16* qg, const lh_bf16* kg,
                      const lh_bf16* vg, lh_bf16* og, lh_bf16* og_lo, float* lse,
                      void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(qg, kg, vg, og, lse)) return LH_ERR_INVALID_ARGUMENT;
  if (og_lo && !aligned(og_lo)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  return cu(lh_launch_attn_fwd(D.B * D.H, D.S, D.d, D.scale, qg, kg, vg, og, og_lo, lse,
                               D.status, (cudaStream_t)stream));
}

lh_status lh_attn_bwd(const lh_config* cfg, const lh_bf16* qg, const lh_bf16* kg,
                      const lh_bf16* vg, const lh_bf16* og, const lh_bf16* og_lo,
                      const float* lse, const lh_bf16* dog, lh_bf16* dqg, lh_bf16* dkg,
                      lh_bf16* dvg, void* ws, size_t ws_bytes, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(qg, kg, vg, og, lse, dog, dqg, dkg, dvg, ws)) return LH_ERR_INVALID_ARGUMENT;
  if (og_lo && !aligned(og_lo)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  const BwdWs b = bwd_layout(D);
  if (ws_bytes < b.total) return LH_ERR_WORKSPACE;
  const cudaStream_t st = (cudaStream_t)stream;
  float* delta = at<float>(ws, b.delta);
  LH_TRY(cu(lh_launch_attn_delta(D.B * D.H, D.S, D.d, og, og_lo, dog, delta, st)));
  return cu(lh_launch_attn_bwd(D.B * D.H, D.S, D.d, D.scale, qg, kg, vg, dog, lse, delta, dqg,
                               dkg, dvg, D.status, st, 3));
}

lh_status lh_attn_bwd_dkdv(const lh_config* cfg, const lh_bf16* qg, const lh_bf16* kg,
                           const lh_bf16* vg, const lh_bf16* dog, const float* lse,
                           const float* delta, lh_bf16* dkg, lh_bf16* dvg, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(qg, kg, vg, dog, lse, delta, dkg, dvg)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  return cu(lh_launch_attn_bwd(D.B * D.H, D.S, D.d, D.scale, qg, kg, vg, dog, lse, delta, nullptr,
                               dkg, dvg, D.status, (cudaStream_t)stream, 1));
}

lh_status lh_attn_bwd_dq(const lh_config* cfg, const lh_bf16* qg, const lh_bf16* kg,
                         const lh_bf16* vg, const lh_bf16* dog, const float* lse,
                         const float* delta, lh_bf16* dqg, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(qg, kg, vg, dog, lse, delta, dqg)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  return cu(lh_launch_attn_bwd(D.B * D.H, D.S, D.d, D.scale, qg, kg, vg, dog, lse, delta, dqg,
                               nullptr, nullptr, D.status, (cudaStream_t)stream, 2));
}

// ---- ring steps (context parallelism) --------------------------------------

namespace {
// Mode and flags of one ring step; the accumulators a step reads or keeps
// must be given, the outputs a closing step writes must be given.
lh_status ring_args(int32_t mode, int32_t first, int32_t last) {
  if (mode != LH_BLOCK_DIAG && mode != LH_BLOCK_FULL) return LH_ERR_INVALID_ARGUMENT;
  if ((first != 0 && first != 1) || (last != 0 && last != 1)) return LH_ERR_INVALID_ARGUMENT;
  return LH_OK;
}
inline bool acc_ok(int32_t first, int32_t last, const void* a) {
  return (first && last) || (a != nullptr && aligned(a));
}
inline bool out_ok(int32_t last, const void* o) { return !last || (o != nullptr && aligned(o)); }
}  // namespace

lh_status lh_attn_fwd_block(const lh_config* cfg, int32_t mode, int32_t first, int32_t last,
                            const lh_bf16* qg, const lh_bf16* kg, const lh_bf16* vg,
                            float* o_acc, float* lse2_acc, lh_bf16* og, lh_bf16* og_lo,
                            float* lse, void* stream) {
  LH_TRY(check(cfg));
  LH_TRY(ring_args(mode, first, last));
  if (!all_aligned(qg, kg, vg)) return LH_ERR_INVALID_ARGUMENT;
  if (!acc_ok(first, last, o_acc) || !acc_ok(first, last, lse2_acc)) return LH_ERR_INVALID_ARGUMENT;
  if (!out_ok(last, og) || !out_ok(last, lse) || (og_lo && !aligned(og_lo)))
    return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  return cu(lh_launch_attn_fwd(D.B * D.H, D.S, D.d, D.scale, qg, kg, vg, og, last ? og_lo : nullptr,
                               lse, D.status, (cudaStream_t)stream, mode == LH_BLOCK_FULL, first,
                               last, o_acc, lse2_acc));
}

lh_status lh_attn_bwd_dkdv_block(const lh_config* cfg, int32_t mode, int32_t first,
                                 int32_t last, const lh_bf16* qg, const lh_bf16* kg,
                                 const lh_bf16* vg, const lh_bf16* dog, const float* lse,
                                 const float* delta, float* dk_acc, float* dv_acc, lh_bf16* dkg,
                                 lh_bf16* dvg, void* stream) {
  LH_TRY(check(cfg));
  LH_TRY(ring_args(mode, first, last));
  if (!all_aligned(qg, kg, vg, dog, lse, delta)) return LH_ERR_INVALID_ARGUMENT;
  if (!acc_ok(first, last, dk_acc) || !acc_ok(first, last, dv_acc)) return LH_ERR_INVALID_ARGUMENT;
  if (!out_ok(last, dkg) || !out_ok(last, dvg)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  LhRingStep rs;
  rs.full = mode == LH_BLOCK_FULL;
  rs.kv_first = first;
  rs.kv_last = last;
  rs.dk_acc = dk_acc;
  rs.dv_acc = dv_acc;
  return cu(lh_launch_attn_bwd(D.B * D.H, D.S, D.d, D.scale, qg, kg, vg, dog, lse, delta, nullptr,
                               dkg, dvg, D.status, (cudaStream_t)stream, 1, &rs));
}

lh_status lh_attn_bwd_dq_block(const lh_config* cfg, int32_t mode, int32_t first, int32_t last,
                               const lh_bf16* qg, const lh_bf16* kg, const lh_bf16* vg,
                               const lh_bf16* dog, const float* lse, const float* delta,
                               float* dq_acc, lh_bf16* dqg, void* stream) {
  LH_TRY(check(cfg));
  LH_TRY(ring_args(mode, first, last));
  if (!all_aligned(qg, kg, vg, dog, lse, delta)) return LH_ERR_INVALID_ARGUMENT;
  if (!acc_ok(first, last, dq_acc) || !out_ok(last, dqg)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  LhRingStep rs;
  rs.full = mode == LH_BLOCK_FULL;
  rs.q_first = first;
  rs.q_last = last;
  rs.dq_acc = dq_acc;
  return cu(lh_launch_attn_bwd(D.B * D.H, D.S, D.d, D.scale, qg, kg, vg, dog, lse, delta, dqg,
                               nullptr, nullptr, D.status, (cudaStream_t)stream, 2, &rs));
}

lh_status lh_scatter(const lh_config* cfg, const lh_bf16* og, const int32_t* slot_map,
                     lh_bf16* o, void* ws, size_t ws_bytes, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(og, slot_map, o)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  if (cfg->scatter_mode == 1) {
    if (!all_aligned(ws)) return LH_ERR_INVALID_ARGUMENT;
    if (ws_bytes < lh_scatter_atomic_ws_bytes(D)) return LH_ERR_WORKSPACE;
    return cu(lh_launch_scatter_atomic(D, og, slot_map, o, ws, (cudaStream_t)stream, nullptr));
  }
  return cu(lh_launch_scatter(D, og, slot_map, o, (cudaStream_t)stream));
}

lh_status lh_scatter_bwd(const lh_config* cfg, const lh_bf16* dout, const lh_bf16* og,
                         const lh_bf16* og_lo, const int32_t* sel_idx, lh_bf16* dog,
                         float* delta, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(dout, og, sel_idx, dog, delta)) return LH_ERR_INVALID_ARGUMENT;
  if (og_lo && !aligned(og_lo)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  return cu(lh_launch_scatter_bwd(D, dout, og, og_lo, sel_idx, dog, delta, (cudaStream_t)stream));
}

lh_status lh_gather_bwd(const lh_config* cfg, const lh_bf16* dqg, const lh_bf16* dkg,
                        const lh_bf16* dvg, const int32_t* slot_map, lh_bf16* dq, lh_bf16* dk,
                        lh_bf16* dv, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(dqg, dkg, dvg, slot_map, dq, dk, dv)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  return cu(lh_launch_gather_bwd(D, dqg, dkg, dvg, slot_map, dq, dk, dv, (cudaStream_t)stream));
}

lh_status lh_forward(const lh_config* cfg, const lh_bf16* q, const lh_bf16* k,
                     const lh_bf16* v, lh_bf16* o, void* saved, size_t saved_bytes, void* ws,
                     size_t ws_bytes, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(q, k, v, o, saved, ws)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  const FwdWs w = fwd_layout(D, cfg->scatter_mode);
  const Saved s = saved_layout(D);
  if (ws_bytes < w.total || saved_bytes < s.total) return LH_ERR_WORKSPACE;
  const cudaStream_t st = (cudaStream_t)stream;
  int32_t* sel_idx = at<int32_t>(saved, s.off[0]);
  int32_t* slot_map = at<int32_t>(saved, s.off[1]);
  lh_bf16* qg = at<lh_bf16>(saved, s.off[2]);
  lh_bf16* kg = at<lh_bf16>(saved, s.off[3]);
  lh_bf16* vg = at<lh_bf16>(saved, s.off[4]);
  lh_bf16* og = at<lh_bf16>(saved, s.off[5]);
  lh_bf16* og_lo = at<lh_bf16>(saved, s.off[6]);
  float* lse = at<float>(saved, s.off[7]);
  lh_bf16* q_lv = at<lh_bf16>(ws, w.q_lv);
  lh_bf16* k_lv = at<lh_bf16>(ws, w.k_lv);
  lh_bf16* v_lv = at<lh_bf16>(ws, w.v_lv);
  float* qk = at<float>(ws, w.qk);
  float* kq = at<float>(ws, w.kq);
  LH_TRY(cu(lh_launch_pyramid(D, q, k, v, q_lv, k_lv, v_lv, qk, kq, st)));
  LH_TRY(cu(lh_launch_select(D, qk, kq, sel_idx, slot_map, at<void>(ws, w.select), st, nullptr)));
  LH_TRY(cu(lh_launch_gather(D, q, k, v, q_lv, k_lv, v_lv, sel_idx, qg, kg, vg, st)));
  LH_TRY(cu(lh_launch_attn_fwd(D.B * D.H, D.S, D.d, D.scale, qg, kg, vg, og, og_lo, lse, D.status,
                               st)));
  if (cfg->scatter_mode == 1)
    return cu(lh_launch_scatter_atomic(D, og, slot_map, o, at<void>(ws, w.atomic), st, nullptr));
  return cu(lh_launch_scatter(D, og, slot_map, o, st));
}

// ---- the layer in halves around its attention ------------------------------

lh_status lh_forward_gather(const lh_config* cfg, const lh_bf16* q, const lh_bf16* k,
                            const lh_bf16* v, void* saved, size_t saved_bytes, void* ws,
                            size_t ws_bytes, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(q, k, v, saved, ws)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  const FwdWs w = fwd_layout(D, cfg->scatter_mode);
  const Saved s = saved_layout(D);
  if (ws_bytes < w.total || saved_bytes < s.total) return LH_ERR_WORKSPACE;
  const cudaStream_t st = (cudaStream_t)stream;
  int32_t* sel_idx = at<int32_t>(saved, s.off[0]);
  int32_t* slot_map = at<int32_t>(saved, s.off[1]);
  lh_bf16* q_lv = at<lh_bf16>(ws, w.q_lv);
  lh_bf16* k_lv = at<lh_bf16>(ws, w.k_lv);
  lh_bf16* v_lv = at<lh_bf16>(ws, w.v_lv);
  float* qk = at<float>(ws, w.qk);
  float* kq = at<float>(ws, w.kq);
  LH_TRY(cu(lh_launch_pyramid(D, q, k, v, q_lv, k_lv, v_lv, qk, kq, st)));
  LH_TRY(cu(lh_launch_select(D, qk, kq, sel_idx, slot_map, at<void>(ws, w.select), st, nullptr)));
  return cu(lh_launch_gather(D, q, k, v, q_lv, k_lv, v_lv, sel_idx, at<lh_bf16>(saved, s.off[2]),
                             at<lh_bf16>(saved, s.off[3]), at<lh_bf16>(saved, s.off[4]), st));
}

lh_status lh_forward_scatter(const lh_config* cfg, const void* saved, size_t saved_bytes,
                             lh_bf16* o, void* ws, size_t ws_bytes, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(saved, o, ws)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  const FwdWs w = fwd_layout(D, cfg->scatter_mode);
  const Saved s = saved_layout(D);
  if (ws_bytes < w.total || saved_bytes < s.total) return LH_ERR_WORKSPACE;
  const cudaStream_t st = (cudaStream_t)stream;
  const lh_bf16* og = at<lh_bf16>(saved, s.off[5]);
  const int32_t* slot_map = at<int32_t>(saved, s.off[1]);
  if (cfg->scatter_mode == 1)
    return cu(lh_launch_scatter_atomic(D, og, slot_map, o, at<void>(ws, w.atomic), st, nullptr));
  return cu(lh_launch_scatter(D, og, slot_map, o, st));
}

lh_status lh_backward_scatter(const lh_config* cfg, const void* saved, size_t saved_bytes,
                              const lh_bf16* dout, void* ws, size_t ws_bytes, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(saved, dout, ws)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  const Saved s = saved_layout(D);
  const BwdWs b = bwd_layout(D);
  if (saved_bytes < s.total || ws_bytes < b.total) return LH_ERR_WORKSPACE;
  return cu(lh_launch_scatter_bwd(D, dout, at<lh_bf16>(saved, s.off[5]),
                                  at<lh_bf16>(saved, s.off[6]), at<int32_t>(saved, s.off[0]),
                                  at<lh_bf16>(ws, b.dog), at<float>(ws, b.delta),
                                  (cudaStream_t)stream));
}

lh_status lh_backward_gather(const lh_config* cfg, const void* saved, size_t saved_bytes,
                             const void* ws, size_t ws_bytes, lh_bf16* dq, lh_bf16* dk,
                             lh_bf16* dv, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(saved, ws, dq, dk, dv)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  const Saved s = saved_layout(D);
  const BwdWs b = bwd_layout(D);
  if (saved_bytes < s.total || ws_bytes < b.total) return LH_ERR_WORKSPACE;
  return cu(lh_launch_gather_bwd(D, at<lh_bf16>(ws, b.dqg), at<lh_bf16>(ws, b.dkg),
                                 at<lh_bf16>(ws, b.dvg), at<int32_t>(saved, s.off[1]), dq, dk, dv,
                                 (cudaStream_t)stream));
}

lh_status lh_backward(const lh_config* cfg, const void* saved, size_t saved_bytes,
                      const lh_bf16* dout, lh_bf16* dq, lh_bf16* dk, lh_bf16* dv, void* ws,
                      size_t ws_bytes, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(saved, dout, dq, dk, dv, ws)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  const Saved s = saved_layout(D);
  const BwdWs b = bwd_layout(D);
  if (saved_bytes < s.total || ws_bytes < b.total) return LH_ERR_WORKSPACE;
  const cudaStream_t st = (cudaStream_t)stream;
  const int32_t* sel_idx = at<int32_t>(saved, s.off[0]);
  const int32_t* slot_map = at<int32_t>(saved, s.off[1]);
  const lh_bf16* qg = at<lh_bf16>(saved, s.off[2]);
  const lh_bf16* kg = at<lh_bf16>(saved, s.off[3]);
  const lh_bf16* vg = at<lh_bf16>(saved, s.off[4]);
  const lh_bf16* og = at<lh_bf16>(saved, s.off[5]);
  const lh_bf16* og_lo = at<lh_bf16>(saved, s.off[6]);
  const float* lse = at<float>(saved, s.off[7]);
  lh_bf16* dog = at<lh_bf16>(ws, b.dog);
  float* delta = at<float>(ws, b.delta);
  lh_bf16* dqg = at<lh_bf16>(ws, b.dqg);
  lh_bf16* dkg = at<lh_bf16>(ws, b.dkg);
  lh_bf16* dvg = at<lh_bf16>(ws, b.dvg);
  LH_TRY(cu(lh_launch_scatter_bwd(D, dout, og, og_lo, sel_idx, dog, delta, st)));
  LH_TRY(cu(lh_launch_attn_bwd(D.B * D.H, D.S, D.d, D.scale, qg, kg, vg, dog, lse, delta, dqg,
                               dkg, dvg, D.status, st, 3)));
  return cu(lh_launch_gather_bwd(D, dqg, dkg, dvg, slot_map, dq, dk, dv, st));
}

size_t lh_gemm_ws_bytes(int64_t M, int64_t N, int32_t splits) {
  if (M < 1 || N < 1 || splits < 1) return 0;
  return lh_gemm_partial_bytes(M, N, splits);
}

lh_status lh_gemm(int64_t M, int64_t N, int32_t npairs, const lh_gemm_operand* ops, int32_t a_mn,
                  int32_t b_mn, lh_bf16* c, int64_t ldc, int32_t splits, void* ws,
                  size_t ws_bytes, void* stream) {
  if (!ops || !c || npairs < 1 || npairs > 3 || M < 1 || N < 1 || splits < 1) return LH_ERR_INVALID_ARGUMENT;
  if (M >= (1LL << 31) || N >= (1LL << 31) || (N % 8) || ldc < N || (ldc % 8)) return LH_ERR_INVALID_ARGUMENT;
  if ((a_mn != 0 && a_mn != 1) || (b_mn != 0 && b_mn != 1)) return LH_ERR_INVALID_ARGUMENT;
  if (!all_aligned(c)) return LH_ERR_INVALID_ARGUMENT;
  int64_t total = 0;
  for (int i = 0; i < npairs; ++i) {
    const lh_gemm_operand& o = ops[i];
    if (!o.a || !o.b || o.k < 1 || (o.k % 8) || o.k >= (1LL << 31)) return LH_ERR_INVALID_ARGUMENT;
    if (!all_aligned(o.a, o.b) || (o.lda % 8) || (o.ldb % 8)) return LH_ERR_INVALID_ARGUMENT;
    if (o.lda < (a_mn ? M : o.k) || o.ldb < (b_mn ? N : o.k)) return LH_ERR_INVALID_ARGUMENT;
    total += (o.k + 63) / 64;
  }
  if (splits > total) splits = (int32_t)total;
  if (splits > 1 && (!ws || ws_bytes < lh_gemm_partial_bytes(M, N, splits) || !all_aligned(ws)))
    return LH_ERR_WORKSPACE;
  int* st = status_ptr();
  if (!st) return LH_ERR_CUDA;
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return cu(lh_launch_gemm(M, N, npairs, ops, a_mn, b_mn, c, ldc, splits, ws, st, sms,
                           (cudaStream_t)stream, nullptr));
}

lh_status lh_check_wait_timeout(void* stream) {
  int* p = status_ptr();
  if (!p) return LH_ERR_CUDA;
  return cu(lh_launch_wait_timeout_check(p, LH_WAIT_TIMEOUT_CHECK_DETAIL, (cudaStream_t)stream));
}

lh_status lh_get_device_status(void* stream, int32_t* detail) {
  int* p = status_ptr();
  if (!p) return LH_ERR_CUDA;
  int h[2] = {0, 0};
  const cudaStream_t st = (cudaStream_t)stream;
  if (cudaMemcpyAsync(h, p, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess) return LH_ERR_CUDA;
  if (cudaMemsetAsync(p, 0, sizeof(h), st) != cudaSuccess) return LH_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return LH_ERR_CUDA;
  if (detail) *detail = h[1];
  return (lh_status)h[0];
}

const char* lh_status_string(lh_status s) {
  switch (s) {
    case LH_OK: return "ok";
    case LH_ERR_INVALID_ARGUMENT: return "invalid argument";
    case LH_ERR_UNSUPPORTED: return "unsupported configuration";
    case LH_ERR_WORKSPACE: return "workspace or saved buffer too small";
    case LH_ERR_CUDA: return "CUDA launch or driver error";
    case LH_ERR_DEVICE_TIMEOUT: return "device-side wait timed out";
    case LH_ERR_DEVICE_BOUNDS: return "device-side index check failed";
  }
  return "unknown status";
}

// ---------------------------------------------------------------------------
// lh_score_topk without a caller workspace.  The selection scratch (digit
// histograms, per-head threshold state, per-block counts) lives in this
// fixed device array instead; every device that loads the library keeps it
// until the process exits.  Host code must not hand the array's name to a
// kernel (on the host it names a stand-in, not device memory): the device
// address is looked up with cudaGetSymbolAddress, with the device current,
// and that pointer is what the kernels get.
constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;  // 8 MiB
static __device__ __align__(256) unsigned char g_topk_scratch[kNoAllocScratchBytes];

// Looked up on every call (see status_ptr): thread-safe, and never stale.
static void* topk_scratch_ptr() {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_topk_scratch) != cudaSuccess) return nullptr;
  return p;
}

lh_status lh_score_topk_noalloc(const lh_config* cfg, const float* qk, const float* kq,
                                int32_t* sel_idx, int32_t* slot_map, void* stream) {
  LH_TRY(check(cfg));
  if (!all_aligned(qk, kq, sel_idx, slot_map)) return LH_ERR_INVALID_ARGUMENT;
  const LhDims D = launch_dims(cfg);
  if (!D.status) return LH_ERR_CUDA;
  if (lh_select_ws_bytes(D) > kNoAllocScratchBytes) return LH_ERR_WORKSPACE;
  void* scratch = topk_scratch_ptr();
  if (!scratch) return LH_ERR_CUDA;
  // lh_launch_select zeroes the histograms it accumulates into before use;
  // the state and block counts are written before they are read.
  return cu(lh_launch_select(D, qk, kq, sel_idx, slot_map, scratch, (cudaStream_t)stream,
                             nullptr));
}

size_t lh_score_topk_noalloc_max_bytes(void) { return kNoAllocScratchBytes; }

int32_t lh_forward_launches(const lh_config* cfg) {
  if (check(cfg) != LH_OK) return -1;
  const LhDims D = dims(cfg);
  // kernels only (the memsets of the scratch are copy-engine work, not counted)
  // hist/find pairs (one fused chunk kernel when stratified) + order count/scan/emit
  const int select = D.select_mode == 2 ? 1 + 3 : (D.n_cand > 0 ? 12 + 3 : 1 + 3);
  const int scatter = cfg->scatter_mode == 1 ? 2 : 1;
  return 1 + select + 1 + 1 + scatter;
}

int32_t lh_backward_launches(const lh_config* cfg) {
  if (check(cfg) != LH_OK) return -1;
  return 1 + 2 + 1;  // scatter_bwd, attention dK/dV and dQ, gather_bwd
}

}  // extern "C"
