// Host side of the C ABI declared in include/vsa.h: validation, workspace
// layout, plan (tensor-map descriptors), launches and error reporting.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <new>

#include "../../include/vsa.h"
#include "vsa_common.cuh"

// State of vsa_run_host, created by its first call on a plan: device copies
// of the inputs and results, a plan (and workspace) over one (batch, head)
// slice, two copy streams and the events that chain the slices.
struct HostPath {
  vsa_plan_s* sub;
  void* sub_ws;
  char* dbuf;       // device copies: q, k, v, gate_c, gate_f, out, idx, cnt
  size_t off[8];    // offsets of the eight arrays in dbuf
  size_t slice[8];  // bytes of one (batch, head) slice of each
  cudaStream_t s_in, s_out;
  cudaEvent_t e_start, e_end;
  cudaEvent_t* e_in;   // per slice: inputs on the device
  cudaEvent_t* e_out;  // per slice: results on the device
};

struct vsa_plan_s {
  // Serialises the host-side work of calls on this plan (tensor-map encoding,
  // launches, the recorded stream), so that two threads sharing a plan never
  // launch with a map encoded for the other thread's q or out. The workspace
  // itself is still one per plan: work of calls on different streams without
  // ordering between them races on it on the device.
  std::mutex mu;
  vsa_config cfg;
  int BH, N, C, kcap;
  char* ws;
  vsa_workspace_layout_t lay;
  CUtensorMap tm_k, tm_v;   // maps over the cube-major copies in the workspace
  CUtensorMap tm_qc;        // map over q's cube-major copy (written by the backward pass's gather)
  CUtensorMap tm_qs, tm_ks, tm_vs, tm_ps;  // maps over the coarse operands' bf16 terms
  CUtensorMap tm_out;       // output map, encoded for the output pointer tm_out_for
  const void* tm_out_for;
  int cube_copies;          // also write q's cube-major copy (inspection)
  int num_sms;
  cudaStream_t last_stream;
  uint64_t wait_ns;
  int debug_stall;
  int timing;        // record stage events
  int timed_runs;    // runs recorded since timing was enabled
  cudaEvent_t* ev;     // stage events of the forward: 4 per run, for the last `ring` runs
  int ring;            // runs kept (vsa_set_stage_timing)
  cudaEvent_t* evb;    // backward stage events: 5 per run (prologue, prep + lists + coarse, dQ, dK/dV), `ring` runs
  int timed_bwd;       // backward runs recorded since timing was enabled
  HostPath* host;    // vsa_run_host state (null until its first call)
};

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn get_encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

constexpr int kMaxC = 4096;
// Row pitch of the coarse probabilities' bf16 terms: C rounded up to 8 (16 bytes).
inline size_t coarse_pitch(size_t C) { return (C + 7) / 8 * 8; }
constexpr int kMaxTopPKmax = 1024;

vsa_status validate(const vsa_config* c) {
  if (!c) return VSA_ERR_INVALID_ARG;
  if (c->B < 1 || c->heads < 1 || c->T < 4 || c->H < 4 || c->W < 4) return VSA_ERR_SHAPE;
  if (c->T % 4 || c->H % 4 || c->W % 4) return VSA_ERR_SHAPE;
  if (c->D != 64 && c->D != 128) return VSA_ERR_UNSUPPORTED;
  const long long N = (long long)c->T * c->H * c->W;
  const long long C = N / 64;
  if (C > kMaxC) return VSA_ERR_UNSUPPORTED;
  if ((long long)c->B * c->heads * N * c->D >= (1LL << 40)) return VSA_ERR_UNSUPPORTED;
  if ((long long)c->B * c->heads * N >= (1LL << 31)) return VSA_ERR_UNSUPPORTED;  // TMA row coordinates
  if ((long long)c->B * c->heads > 65535) return VSA_ERR_UNSUPPORTED;
  if (c->topk < 0) return VSA_ERR_INVALID_ARG;
  if (c->topk > 0) {
    if (c->topk > C) return VSA_ERR_INVALID_ARG;
  } else {
    if (!(c->top_p > 0.f && c->top_p <= 1.f)) return VSA_ERR_INVALID_ARG;
    if (c->kmin < 1 || c->kmin > c->kmax || c->kmax > C) return VSA_ERR_INVALID_ARG;
    if (c->kmax > kMaxTopPKmax) return VSA_ERR_UNSUPPORTED;
  }
  return VSA_OK;
}

// with_q_cube: reserve the region of q's cube-major copy (only written when a
// plan asks for it with vsa_set_cube_major_copies; the allocation-free entry
// point never does, so its layout gives the region zero bytes).
void make_layout(const vsa_config* c, vsa_workspace_layout_t* L, bool with_q_cube = true) {
  const size_t BH = (size_t)c->B * c->heads, N = (size_t)c->T * c->H * c->W, C = N / 64, D = c->D;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 1024);
    return o;
  };
  L->q_cube = take(with_q_cube ? BH * N * D * 2 : 0);
  L->k_cube = take(BH * N * D * 2);
  L->v_cube = take(BH * N * D * 2);
  L->q_pool = take(BH * C * D * 4);
  L->k_pool = take(BH * C * D * 4);
  L->v_pool = take(BH * C * D * 4);
  L->o_coarse = take(BH * C * D * 4);
  L->s_coarse = take(BH * C * C * 4);
  L->pool_split = take(9 * BH * C * D * 2);
  L->p_split = take(3 * BH * C * coarse_pitch(C) * 2);
  L->cnt = take(BH * C * 4);
  L->order = take(BH * C * 4);
  L->err = take(16);
  L->total = off;
}

// Regions of the backward pass's workspace (byte offsets).
struct BwdLayout {
  size_t do_cube, qstat, doc, docsplit, dlc, dssplit, dqbar, dkbar, dvbar, bitmap, tcnt, toff, tlist, order_q,
      order_kv, total;
};
void make_bwd_layout(const vsa_config* c, BwdLayout* L) {
  const size_t BH = (size_t)c->B * c->heads, N = (size_t)c->T * c->H * c->W, C = N / 64, D = c->D;
  const size_t kcap = c->topk > 0 ? (size_t)c->topk : (size_t)c->kmax, W32 = (C + 31) / 32;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 1024);
    return o;
  };
  L->do_cube = take(BH * N * D * 2);
  L->qstat = take(BH * C * 128 * 4);
  L->doc = take(BH * C * D * 4);
  L->docsplit = take(3 * BH * C * D * 2);
  L->dlc = take(BH * C * 4);
  L->dssplit = take(3 * BH * C * coarse_pitch(C) * 2);
  L->dqbar = take(BH * C * D * 4);
  L->dkbar = take(BH * C * D * 4);
  L->dvbar = take(BH * C * D * 4);
  L->bitmap = take(BH * C * W32 * 4);
  L->tcnt = take(BH * C * 4);
  L->toff = take(BH * C * 4);
  L->tlist = take(BH * C * kcap * 4);
  L->order_q = take(BH * C * 4);
  L->order_kv = take(BH * C * 4);
  L->total = off;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 2-D map over a cube-major copy: rows of D bf16, 64 x 64 boxes, 128-byte swizzle.
vsa_status encode_cube_map(CUtensorMap* m, void* base, size_t rows, int D) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return VSA_ERR_CUDA;
  cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  cuuint32_t box[2] = {64, 64};
  cuuint32_t es[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? VSA_OK : VSA_ERR_CUDA;
}

// 3-D map over [planes][rows][cols] bf16 (row pitch `pitch` elements), boxes of
// box_rows x 64 columns in the 128-byte swizzle.
vsa_status encode_planes_map(CUtensorMap* m, void* base, size_t cols, size_t pitch, size_t rows, size_t planes,
                             int box_rows) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return VSA_ERR_CUDA;
  cuuint64_t dims[3] = {(cuuint64_t)cols, (cuuint64_t)rows, (cuuint64_t)planes};
  cuuint64_t strides[2] = {(cuuint64_t)pitch * 2, (cuuint64_t)pitch * rows * 2};
  cuuint32_t box[3] = {64, (cuuint32_t)box_rows, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, base, dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? VSA_OK : VSA_ERR_CUDA;
}

// Maps over the bf16 terms of the pooled q, k, v ([3 * BH][C][D] each) and of
// the coarse probabilities ([3 * BH][C][Cp]).
vsa_status encode_coarse_maps(vsa_plan_s* P) {
  const size_t BH = P->BH, C = P->C, D = P->cfg.D, Cp = coarse_pitch(C);
  char* base = P->ws + P->lay.pool_split;
  const size_t tbytes = 3 * BH * C * D * 2;
  vsa_status e = encode_planes_map(&P->tm_qs, base, D, D, C, 3 * BH, 128);
  if (e == VSA_OK) e = encode_planes_map(&P->tm_ks, base + tbytes, D, D, C, 3 * BH, 128);
  if (e == VSA_OK) e = encode_planes_map(&P->tm_vs, base + 2 * tbytes, D, D, C, 3 * BH, 64);
  if (e == VSA_OK) e = encode_planes_map(&P->tm_ps, P->ws + P->lay.p_split, Cp, Cp, C, 3 * BH, 128);
  return e;
}

// 5-D map over a raster output [BH][T][H][W][D] bf16 (out, dq, dk, dv): a box
// is one cube's 4 x 4 x 4 tokens by 64 channels, laid out in shared memory as
// 64 rows (in-cube slot order) of 128 bytes in the 128-byte swizzle.
vsa_status encode_raster_map(CUtensorMap* m, const void* base, const vsa_config& c, int BH) {
  EncodeTiledFn enc = get_encode_fn();
  if (!enc) return VSA_ERR_CUDA;
  const cuuint64_t D = (cuuint64_t)c.D;
  cuuint64_t dims[5] = {D, (cuuint64_t)c.W, (cuuint64_t)c.H, (cuuint64_t)c.T, (cuuint64_t)BH};
  cuuint64_t strides[4] = {D * 2, (cuuint64_t)c.W * D * 2, (cuuint64_t)c.H * c.W * D * 2,
                           (cuuint64_t)c.T * c.H * c.W * D * 2};
  cuuint32_t box[5] = {64, 4, 4, 4, 1};
  cuuint32_t es[5] = {1, 1, 1, 1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(base), dims, strides, box, es,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? VSA_OK : VSA_ERR_CUDA;
}

vsa_status run_common(vsa_plan_t P, const void* q, const void* k, const void* v, const float* gate_c,
                      const float* gate_f, bool select, const int32_t* idx_in, const int32_t* cnt_in, int32_t* idx_out,
                      int32_t* cnt_out, void* out, float* out_coarse, float* out_fine, void* stream,
                      void* o_fine = nullptr, float* lse = nullptr) {
  if (!P || !q || !k || !v || !gate_c || !gate_f) return VSA_ERR_INVALID_ARG;
  if (select && !idx_out) return VSA_ERR_INVALID_ARG;
  if (!select && !idx_in) return VSA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, gate_c, gate_f, idx_in, cnt_in, idx_out, cnt_out, out, out_coarse, out_fine,
                        o_fine, lse};
  for (const void* p : ptrs)
    if (p && !aligned16(p)) return VSA_ERR_ALIGN;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(P->mu);
  P->last_stream = st;
  const vsa_config& c = P->cfg;
  char* ws = P->ws;
  const vsa_workspace_layout_t& L = P->lay;

  vsa::GatherParams gp{};
  gp.src[0] = static_cast<const __nv_bfloat16*>(q);
  gp.src[1] = static_cast<const __nv_bfloat16*>(k);
  gp.src[2] = static_cast<const __nv_bfloat16*>(v);
  if (P->cube_copies) gp.dst[0] = reinterpret_cast<__nv_bfloat16*>(ws + L.q_cube);
  gp.dst[1] = reinterpret_cast<__nv_bfloat16*>(ws + L.k_cube);
  gp.dst[2] = reinterpret_cast<__nv_bfloat16*>(ws + L.v_cube);
  gp.pool[0] = reinterpret_cast<float*>(ws + L.q_pool);
  gp.pool[1] = reinterpret_cast<float*>(ws + L.k_pool);
  gp.pool[2] = reinterpret_cast<float*>(ws + L.v_pool);
  for (int t = 0; t < 3; ++t)
    gp.split[t] = reinterpret_cast<__nv_bfloat16*>(ws + L.pool_split + (size_t)t * 3 * P->BH * P->C * c.D * 2);
  gp.BH = P->BH; gp.C = P->C; gp.H = c.H; gp.W = c.W; gp.N = P->N;
  cudaEvent_t* ev = P->timing ? P->ev + 4 * (P->timed_runs % P->ring) : nullptr;
  if (ev && cudaEventRecord(ev[0], st) != cudaSuccess) return VSA_ERR_CUDA;
  if (vsa::launch_gather(gp, c.D, P->num_sms, st) != cudaSuccess) return VSA_ERR_CUDA;
  if (ev && cudaEventRecord(ev[1], st) != cudaSuccess) return VSA_ERR_CUDA;

  vsa::CoarseParams cp{};
  cp.tm_qs = P->tm_qs; cp.tm_ks = P->tm_ks; cp.tm_vs = P->tm_vs; cp.tm_ps = P->tm_ps;
  cp.psplit = reinterpret_cast<__nv_bfloat16*>(ws + L.p_split);
  cp.p_terms = 2;  // the output product reads hi and mid
  cp.Cp = (int)coarse_pitch(P->C);
  cp.err = reinterpret_cast<int*>(ws + L.err);
  cp.wait_ns = P->wait_ns;
  cp.s = reinterpret_cast<float*>(ws + L.s_coarse);
  cp.oc = reinterpret_cast<float*>(ws + L.o_coarse);
  cp.oc_copy = out_coarse;
  cp.idx = idx_out;
  cp.cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  cp.BH = P->BH; cp.C = P->C; cp.D = c.D; cp.kcap = P->kcap;
  cp.topk = c.topk; cp.top_p = c.top_p; cp.kmin = c.kmin; cp.kmax = c.kmax;
  cp.do_select = select ? 1 : 0;
  cp.scale = 1.0f / std::sqrt((float)c.D);
  if (vsa::launch_coarse(cp, st) != cudaSuccess) return VSA_ERR_CUDA;

  vsa::FineParams fp{};
  fp.tm_k = P->tm_k; fp.tm_v = P->tm_v;
  fp.q = static_cast<const __nv_bfloat16*>(q);
  if (out) {
    if (P->tm_out_for != out) {
      const vsa_status e = encode_raster_map(&P->tm_out, out, c, P->BH);
      if (e != VSA_OK) return e;
      P->tm_out_for = out;
    }
    fp.tm_out = P->tm_out;
  }
  fp.idx = select ? idx_out : idx_in;
  // Top-K rows all hold exactly topk ids: the fine kernel then needs no counts.
  fp.cnt = select ? (P->cfg.topk > 0 ? nullptr : cp.cnt) : cnt_in;
  // Variable counts: work order longest first per head (schedule.cu).
  if (fp.cnt) {
    fp.order = reinterpret_cast<int32_t*>(ws + L.order);
    if (vsa::launch_schedule(fp.cnt, reinterpret_cast<int32_t*>(ws + L.order), P->BH, P->C, P->kcap, st) !=
        cudaSuccess)
      return VSA_ERR_CUDA;
  }
  fp.oc = cp.oc;
  fp.gate_c = gate_c; fp.gate_f = gate_f;
  fp.out = static_cast<__nv_bfloat16*>(out);
  fp.out_fine = out_fine;
  fp.o_fine = static_cast<float*>(o_fine);
  fp.lse = lse;
  fp.err = reinterpret_cast<int*>(ws + L.err);
  fp.wait_ns = P->wait_ns;
  fp.BH = P->BH; fp.C = P->C; fp.H = c.H; fp.W = c.W; fp.N = P->N;
  fp.kcap = P->kcap; fp.n_items = P->BH * P->C;
  fp.scale_log2 = 1.4426950408889634f / std::sqrt((float)c.D);
  fp.debug_stall = P->debug_stall;
  const int grid = fp.n_items < P->num_sms ? fp.n_items : P->num_sms;
  if (ev && cudaEventRecord(ev[2], st) != cudaSuccess) return VSA_ERR_CUDA;
  if (vsa::launch_fine(fp, c.D, grid, st) != cudaSuccess) return VSA_ERR_CUDA;
  if (P->timing) {
    if (cudaEventRecord(ev[3], st) != cudaSuccess) return VSA_ERR_CUDA;
    P->timed_runs++;
  }

  if (select && cnt_out) {
    if (cudaMemcpyAsync(cnt_out, cp.cnt, (size_t)P->BH * P->C * 4, cudaMemcpyDeviceToDevice, st) != cudaSuccess)
      return VSA_ERR_CUDA;
  }
  return VSA_OK;
}

// Backward pass (see include/vsa.h, vsa_run_backward): the gather (with q's
// cube-major copy) and the coarse stage are recomputed into the plan's
// workspace, then prep, transposed lists, the coarse backward, and the two
// fine backward kernels run with the backward workspace.
vsa_status run_backward(vsa_plan_t P, void* bws, size_t bws_bytes, const void* q, const void* k, const void* v,
                        const float* gate_c, const float* gate_f, const int32_t* idx, const int32_t* cnt,
                        const void* o_fine, const float* lse, const void* dout, void* dq, void* dk, void* dv,
                        float* dgate_c, float* dgate_f, void* stream) {
  if (!P || !bws || !q || !k || !v || !gate_c || !gate_f || !idx || !o_fine || !lse || !dout || !dq || !dk || !dv ||
      !dgate_c || !dgate_f)
    return VSA_ERR_INVALID_ARG;
  const void* ptrs[] = {q, k, v, gate_c, gate_f, idx, cnt, o_fine, lse, dout, dq, dk, dv, dgate_c, dgate_f};
  for (const void* x : ptrs)
    if (x && !aligned16(x)) return VSA_ERR_ALIGN;
  if (reinterpret_cast<uintptr_t>(bws) & 255u) return VSA_ERR_ALIGN;
  BwdLayout BL;
  make_bwd_layout(&P->cfg, &BL);
  if (bws_bytes < BL.total) return VSA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  std::lock_guard<std::mutex> lock(P->mu);
  P->last_stream = st;
  const vsa_config& c = P->cfg;
  const int D = c.D;
  char* ws = P->ws;
  char* bw = static_cast<char*>(bws);
  const vsa_workspace_layout_t& L = P->lay;
  const bool timing = P->timing && P->evb;
  cudaEvent_t* evb = timing ? P->evb + 5 * (P->timed_bwd % P->ring) : nullptr;
  auto mark = [&](int i) { return !timing || cudaEventRecord(evb[i], st) == cudaSuccess; };

  // 1. gather + pool (with q's cube-major copy), coarse attention without selection
  if (!mark(0)) return VSA_ERR_CUDA;
  vsa::GatherParams gp{};
  gp.src[0] = static_cast<const __nv_bfloat16*>(q);
  gp.src[1] = static_cast<const __nv_bfloat16*>(k);
  gp.src[2] = static_cast<const __nv_bfloat16*>(v);
  gp.dst[0] = reinterpret_cast<__nv_bfloat16*>(ws + L.q_cube);
  gp.dst[1] = reinterpret_cast<__nv_bfloat16*>(ws + L.k_cube);
  gp.dst[2] = reinterpret_cast<__nv_bfloat16*>(ws + L.v_cube);
  gp.pool[0] = reinterpret_cast<float*>(ws + L.q_pool);
  gp.pool[1] = reinterpret_cast<float*>(ws + L.k_pool);
  gp.pool[2] = reinterpret_cast<float*>(ws + L.v_pool);
  for (int t = 0; t < 3; ++t)
    gp.split[t] = reinterpret_cast<__nv_bfloat16*>(ws + L.pool_split + (size_t)t * 3 * P->BH * P->C * D * 2);
  gp.BH = P->BH; gp.C = P->C; gp.H = c.H; gp.W = c.W; gp.N = P->N;
  if (vsa::launch_gather(gp, D, P->num_sms, st) != cudaSuccess) return VSA_ERR_CUDA;
  vsa::CoarseParams cp{};
  cp.tm_qs = P->tm_qs; cp.tm_ks = P->tm_ks; cp.tm_vs = P->tm_vs; cp.tm_ps = P->tm_ps;
  cp.psplit = reinterpret_cast<__nv_bfloat16*>(ws + L.p_split);
  cp.p_terms = 3;  // the coarse backward's products read all three terms
  cp.Cp = (int)coarse_pitch(P->C);
  cp.err = reinterpret_cast<int*>(ws + L.err);
  cp.wait_ns = P->wait_ns;
  cp.s = reinterpret_cast<float*>(ws + L.s_coarse);
  cp.oc = reinterpret_cast<float*>(ws + L.o_coarse);
  cp.cnt = reinterpret_cast<int32_t*>(ws + L.cnt);
  cp.BH = P->BH; cp.C = P->C; cp.D = D; cp.kcap = P->kcap;
  cp.topk = c.topk; cp.top_p = c.top_p; cp.kmin = c.kmin; cp.kmax = c.kmax;
  cp.do_select = 0;
  cp.scale = 1.0f / std::sqrt((float)D);
  if (vsa::launch_coarse(cp, st) != cudaSuccess) return VSA_ERR_CUDA;

  // 2. per-token preparation, transposed lists, coarse backward
  if (!mark(1)) return VSA_ERR_CUDA;
  vsa::PrepParams pp{};
  pp.dout = static_cast<const __nv_bfloat16*>(dout);
  pp.ofine = static_cast<const float*>(o_fine);
  pp.lse = lse;
  pp.gate_c = gate_c; pp.gate_f = gate_f;
  pp.oc = cp.oc;
  pp.do_cube = reinterpret_cast<__nv_bfloat16*>(bw + BL.do_cube);
  pp.qstat = reinterpret_cast<float*>(bw + BL.qstat);
  pp.doc = reinterpret_cast<float*>(bw + BL.doc);
  pp.docsplit = reinterpret_cast<__nv_bfloat16*>(bw + BL.docsplit);
  pp.dlc = reinterpret_cast<float*>(bw + BL.dlc);
  pp.dgate_c = dgate_c; pp.dgate_f = dgate_f;
  pp.BH = P->BH; pp.C = P->C; pp.H = c.H; pp.W = c.W; pp.N = P->N;
  if (vsa::launch_bwd_prep(pp, D, st) != cudaSuccess) return VSA_ERR_CUDA;
  vsa::TlistParams tp{};
  tp.idx = idx; tp.cnt = cnt;
  tp.bitmap = reinterpret_cast<uint32_t*>(bw + BL.bitmap);
  tp.tcnt = reinterpret_cast<int32_t*>(bw + BL.tcnt);
  tp.toff = reinterpret_cast<int32_t*>(bw + BL.toff);
  tp.tlist = reinterpret_cast<int32_t*>(bw + BL.tlist);
  tp.err = cp.err;
  tp.BH = P->BH; tp.C = P->C; tp.kcap = P->kcap; tp.W32 = (P->C + 31) / 32;
  if (vsa::launch_tlists(tp, st) != cudaSuccess) return VSA_ERR_CUDA;
  vsa::CoarseBwdParams cb{};
  {
    const size_t BHs = P->BH, Cs = P->C, Ds = D, Cp = coarse_pitch(Cs), tbytes = 3 * BHs * Cs * Ds * 2;
    char* pool = ws + L.pool_split;  // [q, k, v][3 terms][BH][C][D]
    char* docs = bw + BL.docsplit;
    char* dss = bw + BL.dssplit;
    vsa_status me = encode_planes_map(&cb.tm_doc128, docs, Ds, Ds, Cs, 3 * BHs, 128);
    if (me == VSA_OK) me = encode_planes_map(&cb.tm_vb128, pool + 2 * tbytes, Ds, Ds, Cs, 3 * BHs, 128);
    if (me == VSA_OK) me = encode_planes_map(&cb.tm_ds128, dss, Cp, Cp, Cs, 3 * BHs, 128);
    if (me == VSA_OK) me = encode_planes_map(&cb.tm_kb64, pool + tbytes, Ds, Ds, Cs, 3 * BHs, 64);
    if (me == VSA_OK) me = encode_planes_map(&cb.tm_qb64, pool, Ds, Ds, Cs, 3 * BHs, 64);
    if (me == VSA_OK) me = encode_planes_map(&cb.tm_doc64, docs, Ds, Ds, Cs, 3 * BHs, 64);
    if (me == VSA_OK) me = encode_planes_map(&cb.tm_ds64, dss, Cp, Cp, Cs, 3 * BHs, 64);
    if (me == VSA_OK) me = encode_planes_map(&cb.tm_p64, ws + L.p_split, Cp, Cp, Cs, 3 * BHs, 64);
    if (me != VSA_OK) return me;
  }
  cb.psplit = cp.psplit;
  cb.dssplit = reinterpret_cast<__nv_bfloat16*>(bw + BL.dssplit);
  cb.Cp = cp.Cp;
  cb.dlc = pp.dlc;
  cb.dqbar = reinterpret_cast<float*>(bw + BL.dqbar);
  cb.dkbar = reinterpret_cast<float*>(bw + BL.dkbar);
  cb.dvbar = reinterpret_cast<float*>(bw + BL.dvbar);
  cb.err = cp.err;
  cb.wait_ns = P->wait_ns;
  cb.BH = P->BH; cb.C = P->C; cb.D = D; cb.scale = cp.scale;
  if (vsa::launch_coarse_bwd(cb, st) != cudaSuccess) return VSA_ERR_CUDA;

  // 3. fine backward: dQ (query-major), then dK / dV (KV-major)
  vsa::BwdFineParams fb{};
  const size_t rows = (size_t)P->BH * P->N;
  vsa_status e = VSA_OK;
  fb.tm_q = P->tm_qc; fb.tm_k = P->tm_k; fb.tm_v = P->tm_v;
  e = encode_cube_map(&fb.tm_do, bw + BL.do_cube, rows, D);
  if (e == VSA_OK) e = encode_raster_map(&fb.tm_out0, dq, c, P->BH);
  if (e != VSA_OK) return e;
  fb.qstat = pp.qstat;
  fb.err = cp.err;
  fb.wait_ns = P->wait_ns;
  fb.BH = P->BH; fb.C = P->C; fb.H = c.H; fb.W = c.W; fb.N = P->N; fb.kcap = P->kcap;
  fb.n_items = P->BH * P->C;
  fb.scale = cp.scale;
  fb.scale_log2 = 1.4426950408889634f / std::sqrt((float)D);
  fb.list = idx; fb.cnt = cnt; fb.off = nullptr;
  fb.cpart0 = cb.dqbar; fb.cpart1 = nullptr;
  fb.order = nullptr;
  if (cnt) {
    fb.order = reinterpret_cast<int32_t*>(bw + BL.order_q);
    if (vsa::launch_schedule(cnt, reinterpret_cast<int32_t*>(bw + BL.order_q), P->BH, P->C, P->kcap, st) !=
        cudaSuccess)
      return VSA_ERR_CUDA;
  }
  const int grid = fb.n_items < P->num_sms ? fb.n_items : P->num_sms;
  if (!mark(2)) return VSA_ERR_CUDA;
  if (vsa::launch_fine_dq(fb, D, grid, st) != cudaSuccess) return VSA_ERR_CUDA;
  e = encode_raster_map(&fb.tm_out0, dk, c, P->BH);
  if (e == VSA_OK) e = encode_raster_map(&fb.tm_out1, dv, c, P->BH);
  if (e != VSA_OK) return e;
  fb.list = tp.tlist; fb.cnt = tp.tcnt; fb.off = tp.toff;
  fb.cpart0 = cb.dkbar; fb.cpart1 = cb.dvbar;
  fb.order = reinterpret_cast<int32_t*>(bw + BL.order_kv);
  if (vsa::launch_schedule(tp.tcnt, reinterpret_cast<int32_t*>(bw + BL.order_kv), P->BH, P->C, P->C, st) !=
      cudaSuccess)
    return VSA_ERR_CUDA;
  if (!mark(3)) return VSA_ERR_CUDA;
  if (vsa::launch_fine_dkv(fb, D, grid, st) != cudaSuccess) return VSA_ERR_CUDA;
  if (!mark(4)) return VSA_ERR_CUDA;
  if (timing) P->timed_bwd++;
  return VSA_OK;
}

}  // namespace

// Releases vsa_run_host state (waits for its streams first).
static void host_path_free(HostPath* H) {
  if (!H) return;
  if (H->s_in) cudaStreamSynchronize(H->s_in);
  if (H->s_out) cudaStreamSynchronize(H->s_out);
  if (H->sub) vsa_plan_destroy(H->sub);
  if (H->sub_ws) cudaFree(H->sub_ws);
  if (H->dbuf) cudaFree(H->dbuf);
  if (H->e_in) {
    for (int i = 0; H->e_in[i]; ++i) cudaEventDestroy(H->e_in[i]);
    delete[] H->e_in;
  }
  if (H->e_out) {
    for (int i = 0; H->e_out[i]; ++i) cudaEventDestroy(H->e_out[i]);
    delete[] H->e_out;
  }
  if (H->e_start) cudaEventDestroy(H->e_start);
  if (H->e_end) cudaEventDestroy(H->e_end);
  if (H->s_in) cudaStreamDestroy(H->s_in);
  if (H->s_out) cudaStreamDestroy(H->s_out);
  delete H;
}

extern "C" {

size_t vsa_workspace_bytes(const vsa_config* cfg) {
  if (validate(cfg) != VSA_OK) return 0;
  vsa_workspace_layout_t L;
  make_layout(cfg, &L);
  return L.total;
}

vsa_status vsa_workspace_layout(const vsa_config* cfg, vsa_workspace_layout_t* layout) {
  if (!layout) return VSA_ERR_INVALID_ARG;
  const vsa_status s = validate(cfg);
  if (s != VSA_OK) return s;
  make_layout(cfg, layout);
  return VSA_OK;
}

vsa_status vsa_plan(vsa_plan_t* out, const vsa_config* cfg, void* workspace, size_t ws_bytes) {
  if (!out) return VSA_ERR_INVALID_ARG;
  *out = nullptr;
  const vsa_status s = validate(cfg);
  if (s != VSA_OK) return s;
  if (!workspace) return VSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(workspace) & 255u) return VSA_ERR_ALIGN;
  vsa_workspace_layout_t L;
  make_layout(cfg, &L);
  if (ws_bytes < L.total) return VSA_ERR_INVALID_ARG;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VSA_ERR_CUDA;
  int major = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return VSA_ERR_CUDA;
  if (major != 10) return VSA_ERR_DEVICE;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return VSA_ERR_CUDA;
  vsa_plan_s* P = new (std::nothrow) vsa_plan_s();
  if (!P) return VSA_ERR_INVALID_ARG;
  P->cfg = *cfg;
  P->N = cfg->T * cfg->H * cfg->W;
  P->C = P->N / 64;
  P->BH = cfg->B * cfg->heads;
  P->kcap = cfg->topk > 0 ? cfg->topk : cfg->kmax;
  P->ws = static_cast<char*>(workspace);
  P->lay = L;
  P->num_sms = sms;
  P->last_stream = nullptr;
  P->wait_ns = 1000000000ull;
  P->debug_stall = 0;
  const size_t rows = (size_t)P->BH * P->N;
  vsa_status e = encode_cube_map(&P->tm_k, P->ws + L.k_cube, rows, cfg->D);
  if (e == VSA_OK) e = encode_cube_map(&P->tm_v, P->ws + L.v_cube, rows, cfg->D);
  if (e == VSA_OK) e = encode_cube_map(&P->tm_qc, P->ws + L.q_cube, rows, cfg->D);
  if (e == VSA_OK) e = encode_coarse_maps(P);
  if (e == VSA_OK && cudaMemset(P->ws + L.err, 0, 16) != cudaSuccess) e = VSA_ERR_CUDA;
  if (e != VSA_OK) {
    delete P;
    return e;
  }
  *out = P;
  return VSA_OK;
}

vsa_status vsa_run(vsa_plan_t plan, const void* q, const void* k, const void* v, const float* gate_c,
                   const float* gate_f, void* out, int32_t* idx, int32_t* cnt, void* stream) {
  if (!out) return VSA_ERR_INVALID_ARG;
  return run_common(plan, q, k, v, gate_c, gate_f, true, nullptr, nullptr, idx, cnt, out, nullptr, nullptr, stream);
}

vsa_status vsa_run_fixed_idx(vsa_plan_t plan, const void* q, const void* k, const void* v, const float* gate_c,
                             const float* gate_f, const int32_t* idx_in, const int32_t* cnt_in, void* out,
                             float* out_coarse, float* out_fine, void* stream) {
  return run_common(plan, q, k, v, gate_c, gate_f, false, idx_in, cnt_in, nullptr, nullptr, out, out_coarse, out_fine,
                    stream);
}

vsa_status vsa_run_train(vsa_plan_t plan, const void* q, const void* k, const void* v, const float* gate_c,
                         const float* gate_f, void* out, int32_t* idx, int32_t* cnt, void* o_fine, float* lse,
                         void* stream) {
  if (!out || !o_fine || !lse) return VSA_ERR_INVALID_ARG;
  return run_common(plan, q, k, v, gate_c, gate_f, true, nullptr, nullptr, idx, cnt, out, nullptr, nullptr, stream,
                    o_fine, lse);
}

size_t vsa_backward_workspace_bytes(const vsa_config* cfg) {
  if (validate(cfg) != VSA_OK) return 0;
  BwdLayout L;
  make_bwd_layout(cfg, &L);
  return L.total;
}

vsa_status vsa_run_backward(vsa_plan_t plan, void* bwd_workspace, size_t bwd_bytes, const void* q, const void* k,
                            const void* v, const float* gate_c, const float* gate_f, const int32_t* idx,
                            const int32_t* cnt, const void* o_fine, const float* lse, const void* dout, void* dq,
                            void* dk, void* dv, float* dgate_c, float* dgate_f, void* stream) {
  return run_backward(plan, bwd_workspace, bwd_bytes, q, k, v, gate_c, gate_f, idx, cnt, o_fine, lse, dout, dq, dk,
                      dv, dgate_c, dgate_f, stream);
}

vsa_status vsa_backward_stage_times_history(vsa_plan_t plan, float* ms, int max_runs, int* n_runs) {
  if (!plan || !ms || !n_runs || max_runs < 1 || !plan->timing || plan->timed_bwd == 0) return VSA_ERR_INVALID_ARG;
  const int kept = plan->timed_bwd < plan->ring ? plan->timed_bwd : plan->ring;
  const int n = kept < max_runs ? kept : max_runs;
  const int last = plan->timed_bwd - 1;
  if (cudaEventSynchronize(plan->evb[5 * (last % plan->ring) + 4]) != cudaSuccess) return VSA_ERR_CUDA;
  for (int r = 0; r < n; ++r) {
    const cudaEvent_t* e = plan->evb + 5 * ((last - (n - 1) + r) % plan->ring);
    for (int i = 0; i < 4; ++i)
      if (cudaEventElapsedTime(&ms[4 * r + i], e[i], e[i + 1]) != cudaSuccess) return VSA_ERR_CUDA;
  }
  *n_runs = n;
  return VSA_OK;
}

vsa_status vsa_backward_stage_times(vsa_plan_t plan, float* ms) {
  int n = 0;
  return vsa_backward_stage_times_history(plan, ms, 1, &n);
}

vsa_status vsa_run_host(vsa_plan_t plan, const void* q, const void* k, const void* v, const float* gate_c,
                        const float* gate_f, void* out, int32_t* idx, int32_t* cnt, void* stream) {
  if (!plan || !q || !k || !v || !gate_c || !gate_f || !out || !idx) return VSA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(plan->mu);
  const int n = plan->BH;
  HostPath* H = plan->host;
  if (!H) {
    H = new (std::nothrow) HostPath();
    if (!H) return VSA_ERR_INVALID_ARG;
    plan->host = H;
    vsa_config sc = plan->cfg;
    sc.B = 1;
    sc.heads = 1;
    const size_t sb = vsa_workspace_bytes(&sc);
    const size_t nd2 = (size_t)plan->N * plan->cfg.D * 2, n4 = (size_t)plan->N * 4;
    const size_t sl[8] = {nd2, nd2, nd2, n4, n4, nd2, (size_t)plan->C * plan->kcap * 4, (size_t)plan->C * 4};
    size_t total = 0;
    for (int a = 0; a < 8; ++a) {
      H->slice[a] = sl[a];
      H->off[a] = total;
      total += align_up(sl[a] * n, 256);
    }
    H->e_in = new (std::nothrow) cudaEvent_t[n + 1]();
    H->e_out = new (std::nothrow) cudaEvent_t[n + 1]();
    bool ok = sb > 0 && H->e_in && H->e_out && cudaMalloc(&H->sub_ws, sb) == cudaSuccess &&
              cudaMalloc(reinterpret_cast<void**>(&H->dbuf), total) == cudaSuccess &&
              cudaStreamCreateWithFlags(&H->s_in, cudaStreamNonBlocking) == cudaSuccess &&
              cudaStreamCreateWithFlags(&H->s_out, cudaStreamNonBlocking) == cudaSuccess &&
              cudaEventCreateWithFlags(&H->e_start, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventCreateWithFlags(&H->e_end, cudaEventDisableTiming) == cudaSuccess;
    for (int i = 0; ok && i < n; ++i)
      ok = cudaEventCreateWithFlags(&H->e_in[i], cudaEventDisableTiming) == cudaSuccess &&
           cudaEventCreateWithFlags(&H->e_out[i], cudaEventDisableTiming) == cudaSuccess;
    vsa_status ps = ok ? vsa_plan(&H->sub, &sc, H->sub_ws, sb) : VSA_ERR_CUDA;
    if (ps != VSA_OK) {
      host_path_free(H);
      plan->host = nullptr;
      return ps;
    }
  }
  H->sub->wait_ns = plan->wait_ns;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // The copies start after the work already on `stream`; `stream` resumes
  // after the last copy back.
  if (cudaEventRecord(H->e_start, st) != cudaSuccess || cudaStreamWaitEvent(H->s_in, H->e_start, 0) != cudaSuccess ||
      cudaStreamWaitEvent(H->s_out, H->e_start, 0) != cudaSuccess)
    return VSA_ERR_CUDA;
  const void* hin[5] = {q, k, v, gate_c, gate_f};
  void* hres[3] = {out, idx, cnt};
  for (int i = 0; i < n; ++i) {
    // slice i in: copy stream 1
    for (int a = 0; a < 5; ++a)
      if (cudaMemcpyAsync(H->dbuf + H->off[a] + i * H->slice[a], static_cast<const char*>(hin[a]) + i * H->slice[a],
                          H->slice[a], cudaMemcpyHostToDevice, H->s_in) != cudaSuccess)
        return VSA_ERR_CUDA;
    if (cudaEventRecord(H->e_in[i], H->s_in) != cudaSuccess || cudaStreamWaitEvent(st, H->e_in[i], 0) != cudaSuccess)
      return VSA_ERR_CUDA;
    // slice i forward: `stream`
    char* d[8];
    for (int a = 0; a < 8; ++a) d[a] = H->dbuf + H->off[a] + i * H->slice[a];
    const vsa_status rs = vsa_run(H->sub, d[0], d[1], d[2], reinterpret_cast<float*>(d[3]),
                                  reinterpret_cast<float*>(d[4]), d[5], reinterpret_cast<int32_t*>(d[6]),
                                  reinterpret_cast<int32_t*>(d[7]), stream);
    if (rs != VSA_OK) return rs;
    if (cudaEventRecord(H->e_out[i], st) != cudaSuccess || cudaStreamWaitEvent(H->s_out, H->e_out[i], 0) != cudaSuccess)
      return VSA_ERR_CUDA;
    // slice i out: copy stream 2
    for (int a = 5; a < 8; ++a)
      if (hres[a - 5] && cudaMemcpyAsync(static_cast<char*>(hres[a - 5]) + i * H->slice[a], d[a], H->slice[a],
                                         cudaMemcpyDeviceToHost, H->s_out) != cudaSuccess)
        return VSA_ERR_CUDA;
  }
  if (cudaEventRecord(H->e_end, H->s_out) != cudaSuccess || cudaStreamWaitEvent(st, H->e_end, 0) != cudaSuccess)
    return VSA_ERR_CUDA;
  plan->last_stream = st;
  return VSA_OK;
}

namespace {
struct CachedPlan {
  vsa_config cfg;
  int device;
  void* ws;
  vsa_plan_t plan;
};
constexpr int kCacheSize = 16;
CachedPlan g_cache[kCacheSize];
int g_cache_n = 0;
std::mutex g_cache_mu;

bool same_cfg(const vsa_config& a, const vsa_config& b) {
  return a.B == b.B && a.heads == b.heads && a.T == b.T && a.H == b.H && a.W == b.W && a.D == b.D &&
         a.topk == b.topk && a.top_p == b.top_p && a.kmin == b.kmin && a.kmax == b.kmax;
}
}  // namespace

vsa_status vsa_forward(const void* q, const void* k, const void* v, const float* gate_c, const float* gate_f, int B,
                       int heads, int T, int H, int W, int D, int topk, float top_p, void* out, int32_t* idx,
                       void* stream) {
  vsa_config cfg{B, heads, T, H, W, D, topk, top_p, 0, 0};
  if (topk == 0) {
    const int C = (T * H * W) / 64;
    cfg.kmax = C < 128 ? C : 128;
    cfg.kmin = cfg.kmax < 4 ? cfg.kmax : 4;
  }
  const vsa_status s = validate(&cfg);
  if (s != VSA_OK) return s;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VSA_ERR_CUDA;
  vsa_plan_t plan = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_cache_mu);
    for (int i = 0; i < g_cache_n; ++i)
      if (g_cache[i].device == dev && same_cfg(g_cache[i].cfg, cfg)) plan = g_cache[i].plan;
    if (!plan) {
      if (g_cache_n == kCacheSize) return VSA_ERR_UNSUPPORTED;
      const size_t bytes = vsa_workspace_bytes(&cfg);
      void* ws = nullptr;
      if (cudaMalloc(&ws, bytes) != cudaSuccess) return VSA_ERR_CUDA;
      const vsa_status ps = vsa_plan(&plan, &cfg, ws, bytes);
      if (ps != VSA_OK) {
        cudaFree(ws);
        return ps;
      }
      g_cache[g_cache_n++] = CachedPlan{cfg, dev, ws, plan};
    }
  }
  return vsa_run(plan, q, k, v, gate_c, gate_f, out, idx, nullptr, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Allocation-free forward (vsa_forward_noalloc). The workspace is this one
// file-scope device array; host code only ever passes its device address,
// looked up once per device with cudaGetSymbolAddress (in host code the
// array's name is a host-side stand-in, not a device address).
namespace {
static __device__ __align__(256) unsigned char g_noalloc_scratch[VSA_NOALLOC_SCRATCH_BYTES];

constexpr int kNoallocMaxDevices = 64;
void* g_noalloc_addr[kNoallocMaxDevices];
std::mutex g_noalloc_mu;

vsa_status noalloc_scratch(int dev, void** out) {
  if (dev < 0 || dev >= kNoallocMaxDevices) return VSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return VSA_ERR_CUDA;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
  return VSA_OK;
}
}  // namespace

extern "C" {

vsa_status vsa_forward_noalloc(const void* q, const void* k, const void* v, const float* gate_c,
                               const float* gate_f, int B, int heads, int T, int H, int W, int D, int topk,
                               float top_p, void* out, int32_t* idx, void* stream) {
  vsa_config cfg{B, heads, T, H, W, D, topk, top_p, 0, 0};
  if (topk == 0) {
    const int C = (T * H * W) / 64;
    cfg.kmax = C < 128 ? C : 128;
    cfg.kmin = cfg.kmax < 4 ? cfg.kmax : 4;
  }
  vsa_status s = validate(&cfg);
  if (s != VSA_OK) return s;
  if (!out || !idx) return VSA_ERR_INVALID_ARG;
  vsa_workspace_layout_t L;
  make_layout(&cfg, &L, /*with_q_cube=*/false);
  if (L.total > VSA_NOALLOC_SCRATCH_BYTES) return VSA_ERR_UNSUPPORTED;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VSA_ERR_CUDA;
  int major = 0, sms = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return VSA_ERR_CUDA;
  if (major != 10) return VSA_ERR_DEVICE;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return VSA_ERR_CUDA;
  void* scratch = nullptr;
  s = noalloc_scratch(dev, &scratch);
  if (s != VSA_OK) return s;
  // A plan on the stack over the static workspace (no heap allocation).
  vsa_plan_s P{};
  P.cfg = cfg;
  P.N = T * H * W;
  P.C = P.N / 64;
  P.BH = B * heads;
  P.kcap = cfg.topk > 0 ? cfg.topk : cfg.kmax;
  P.ws = static_cast<char*>(scratch);
  P.lay = L;
  P.num_sms = sms;
  P.wait_ns = 1000000000ull;
  const size_t rows = (size_t)P.BH * P.N;
  s = encode_cube_map(&P.tm_k, P.ws + L.k_cube, rows, D);
  if (s == VSA_OK) s = encode_cube_map(&P.tm_v, P.ws + L.v_cube, rows, D);
  if (s == VSA_OK) s = encode_coarse_maps(&P);
  if (s != VSA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(P.ws + L.err, 0, 16, st) != cudaSuccess) return VSA_ERR_CUDA;
  return run_common(&P, q, k, v, gate_c, gate_f, true, nullptr, nullptr, idx, nullptr, out, nullptr, nullptr,
                    stream);
}

vsa_status vsa_check(vsa_plan_t plan) {
  if (!plan) return VSA_ERR_INVALID_ARG;
  if (plan->host && plan->host->sub) {
    const vsa_status hs = vsa_check(plan->host->sub);
    if (hs != VSA_OK) return hs;
  }
  cudaStream_t last;
  {
    std::lock_guard<std::mutex> lock(plan->mu);
    last = plan->last_stream;
  }
  if (cudaStreamSynchronize(last) != cudaSuccess) return VSA_ERR_CUDA;
  int err = 0;
  int* dev_err = reinterpret_cast<int*>(plan->ws + plan->lay.err);
  if (cudaMemcpy(&err, dev_err, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return VSA_ERR_CUDA;
  if (err) {
    if (cudaMemset(dev_err, 0, sizeof(int)) != cudaSuccess) return VSA_ERR_CUDA;
  }
  if (err & vsa::kErrTimeout) return VSA_ERR_TIMEOUT;
  if (err & vsa::kErrBadIndex) return VSA_ERR_INVALID_ARG;
  return VSA_OK;
}

void vsa_plan_destroy(vsa_plan_t plan) {
  if (!plan) return;
  if (plan->ev) {
    for (int i = 0; i < 4 * plan->ring; ++i) cudaEventDestroy(plan->ev[i]);
    delete[] plan->ev;
  }
  if (plan->evb) {
    for (int i = 0; i < 5 * plan->ring; ++i) cudaEventDestroy(plan->evb[i]);
    delete[] plan->evb;
  }
  host_path_free(plan->host);
  delete plan;
}

const char* vsa_status_string(vsa_status s) {
  switch (s) {
    case VSA_OK: return "VSA_OK";
    case VSA_ERR_INVALID_ARG: return "VSA_ERR_INVALID_ARG";
    case VSA_ERR_SHAPE: return "VSA_ERR_SHAPE";
    case VSA_ERR_UNSUPPORTED: return "VSA_ERR_UNSUPPORTED";
    case VSA_ERR_ALIGN: return "VSA_ERR_ALIGN";
    case VSA_ERR_CUDA: return "VSA_ERR_CUDA";
    case VSA_ERR_TIMEOUT: return "VSA_ERR_TIMEOUT";
    case VSA_ERR_DEVICE: return "VSA_ERR_DEVICE";
  }
  return "VSA_ERR_UNKNOWN";
}

vsa_status vsa_set_wait_limit_ns(vsa_plan_t plan, uint64_t limit_ns) {
  if (!plan || limit_ns < 100000ull) return VSA_ERR_INVALID_ARG;
  plan->wait_ns = limit_ns;
  return VSA_OK;
}

vsa_status vsa_set_stage_timing(vsa_plan_t plan, int on) {
  if (!plan) return VSA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(plan->mu);
  const int ring = on <= 0 ? 0 : (on > 4096 ? 4096 : on);
  if (ring > plan->ring) {
    cudaEvent_t* ev = new (std::nothrow) cudaEvent_t[4 * ring]();
    if (!ev) return VSA_ERR_INVALID_ARG;
    for (int i = 0; i < 4 * ring; ++i)
      if (cudaEventCreate(&ev[i]) != cudaSuccess) {
        for (int k = 0; k < i; ++k) cudaEventDestroy(ev[k]);
        delete[] ev;
        return VSA_ERR_CUDA;
      }
    cudaEvent_t* evb = new (std::nothrow) cudaEvent_t[5 * ring]();
    bool ok = evb != nullptr;
    for (int i = 0; ok && i < 5 * ring; ++i)
      if (cudaEventCreate(&evb[i]) != cudaSuccess) {
        for (int k = 0; k < i; ++k) cudaEventDestroy(evb[k]);
        ok = false;
      }
    if (!ok) {
      for (int i = 0; i < 4 * ring; ++i) cudaEventDestroy(ev[i]);
      delete[] ev;
      delete[] evb;
      return VSA_ERR_CUDA;
    }
    if (plan->ev) {
      for (int i = 0; i < 4 * plan->ring; ++i) cudaEventDestroy(plan->ev[i]);
      delete[] plan->ev;
    }
    if (plan->evb) {
      for (int i = 0; i < 5 * plan->ring; ++i) cudaEventDestroy(plan->evb[i]);
      delete[] plan->evb;
    }
    plan->ev = ev;
    plan->evb = evb;
    plan->ring = ring;
  }
  plan->timing = ring > 0 ? 1 : 0;
  plan->timed_runs = 0;
  plan->timed_bwd = 0;
  return VSA_OK;
}

vsa_status vsa_stage_times_history(vsa_plan_t plan, float* ms, int max_runs, int* n_runs) {
  if (!plan || !ms || !n_runs || max_runs < 1 || !plan->timing || plan->timed_runs == 0) return VSA_ERR_INVALID_ARG;
  const int kept = plan->timed_runs < plan->ring ? plan->timed_runs : plan->ring;
  const int n = kept < max_runs ? kept : max_runs;
  const int last = plan->timed_runs - 1;
  if (cudaEventSynchronize(plan->ev[4 * (last % plan->ring) + 3]) != cudaSuccess) return VSA_ERR_CUDA;
  for (int r = 0; r < n; ++r) {
    const cudaEvent_t* e = plan->ev + 4 * ((last - (n - 1) + r) % plan->ring);
    for (int i = 0; i < 3; ++i)
      if (cudaEventElapsedTime(&ms[3 * r + i], e[i], e[i + 1]) != cudaSuccess) return VSA_ERR_CUDA;
  }
  *n_runs = n;
  return VSA_OK;
}

vsa_status vsa_stage_times(vsa_plan_t plan, float* ms) {
  int n = 0;
  return vsa_stage_times_history(plan, ms, 1, &n);
}

int vsa_kernels_per_run(void) { return 5; }  // top-K; variable counts add the schedule kernel

vsa_status vsa_measure_l2_read(const void* buf, size_t bytes, int passes, int* status, void* stream) {
  if (!buf || !status || passes < 1 || bytes < 16384) return VSA_ERR_INVALID_ARG;
  if (!aligned16(buf) || !aligned16(status)) return VSA_ERR_ALIGN;
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return VSA_ERR_CUDA;
  if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return VSA_ERR_CUDA;
  return vsa::launch_l2_read(buf, bytes, passes, status, 2 * sms, reinterpret_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? VSA_OK
             : VSA_ERR_CUDA;
}

vsa_status vsa_set_debug_stall(vsa_plan_t plan, int on) {
  if (!plan) return VSA_ERR_INVALID_ARG;
  plan->debug_stall = on ? 1 : 0;
  return VSA_OK;
}

vsa_status vsa_set_cube_major_copies(vsa_plan_t plan, int on) {
  if (!plan) return VSA_ERR_INVALID_ARG;
  plan->cube_copies = on ? 1 : 0;
  return VSA_OK;
}

}  // extern "C"
