// C ABI of the da2 library: argument checks, workspace layout and stage launches.
#include <cmath>
#include <cstring>

#include <nvtx3/nvToolsExt.h>

#include "checks.cuh"
#include "common.cuh"
#include "split_tiles.cuh"

namespace da2 {
cudaError_t launch_prepare(const Geo& g, const Ws& w, const void* q, const void* k,
                           const void* v, uint8_t* qt, uint8_t* kt, cudaStream_t st);
cudaError_t launch_draft_select(const Geo& g, const Ws& w, const uint8_t* qt, const uint8_t* kt,
                                float* dlog, int np, cudaStream_t st);
cudaError_t launch_attention_tc(const Geo& g, const Ws& w, void* out, cudaStream_t st);
da2_status noalloc_scratch(void** ptr, size_t* bytes);   // da2_noalloc.cu
}  // namespace da2

using namespace da2;

namespace {

constexpr int kMaxBlocks = 4096;
constexpr long kMaxHeads = 65535;   // B * H: the stage kernels put the heads on the grid's y axis

bool pct_ok(int p) { return p >= 0 && p <= 100; }

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

da2_status check_config(const da2_config* c) {
  if (!c) return DA2_ERR_INVALID_ARG;
  if (c->B <= 0 || c->H <= 0 || c->F <= 0 || c->Hf <= 0 || c->Wf <= 0 || c->ph <= 0 || c->pw <= 0)
    return DA2_ERR_INVALID_ARG;
  // each budget on its own first, so that their sums cannot overflow
  if (!pct_ok(c->pct_fp8) || !pct_ok(c->pct_fp4) || !pct_ok(c->pct_mix) ||
      c->pct_fp8 + c->pct_mix + c->pct_fp4 > 100)
    return DA2_ERR_INVALID_ARG;
  if (!(c->sm_scale >= 0.0f) || std::isinf(c->sm_scale)) return DA2_ERR_INVALID_ARG;
  if (!(c->adapt_tau >= 0.0f) || std::isinf(c->adapt_tau)) return DA2_ERR_INVALID_ARG;
  if (c->adapt_tau > 0.0f &&
      (c->pct_fp4_max < c->pct_fp4 || !pct_ok(c->pct_fp4_max) ||
       c->pct_fp8 + c->pct_mix + c->pct_fp4_max > 100))
    return DA2_ERR_INVALID_ARG;
  if (c->flags & ~(DA2_FLAG_EXPORT_SCORES | DA2_FLAG_NO_MASS_CORRECTION | DA2_FLAG_LAYOUT_BTHD |
                   DA2_FLAG_DEBUG_CANARY | DA2_FLAG_TEST_STALL))
    return DA2_ERR_INVALID_ARG;
  if (c->d != 64 && c->d != 128) return DA2_ERR_UNSUPPORTED;
  const long bs = (long)c->ph * c->pw;
  if (bs != 32 && bs != 64 && bs != 128) return DA2_ERR_UNSUPPORTED;
  // in 64-bit steps, each factor bounded before the next product
  const long ny = ((long)c->Hf + c->ph - 1) / c->ph, nx = ((long)c->Wf + c->pw - 1) / c->pw;
  if (c->F > kMaxBlocks || ny > kMaxBlocks || nx > kMaxBlocks) return DA2_ERR_UNSUPPORTED;
  const long N = (long)c->F * ny * nx;
  if (N > kMaxBlocks) return DA2_ERR_UNSUPPORTED;
  if ((long)c->B * c->H > kMaxHeads) return DA2_ERR_UNSUPPORTED;
  if ((long)c->B * c->H * N * N > (1L << 40)) return DA2_ERR_UNSUPPORTED;
  return DA2_OK;
}

// With DA2_FLAG_DEBUG_CANARY every region is followed by a guard of kGuardBytes (its offset
// recorded in *gl when given).
void fill_views(const da2_config* c, da2_views* v, GuardList* gl = nullptr) {
  std::memset(v, 0, sizeof(*v));
  const bool guards = (c->flags & DA2_FLAG_DEBUG_CANARY) != 0;
  if (gl) gl->n = 0;
  v->ny = (c->Hf + c->ph - 1) / c->ph;
  v->nx = (c->Wf + c->pw - 1) / c->pw;
  v->N = c->F * v->ny * v->nx;
  v->bs = c->ph * c->pw;
  v->T = c->F * c->Hf * c->Wf;
  v->Tp = v->N * v->bs;
  const int c8 = (c->pct_fp8 * v->N + 50) / 100;
  const int c8m = ((c->pct_fp8 + c->pct_mix) * v->N + 50) / 100;
  const int ck = ((c->pct_fp8 + c->pct_mix + c->pct_fp4) * v->N + 50) / 100;
  v->n8 = c8;
  v->nm = c8m - c8;
  v->n4 = ck - c8m;
  v->n4max = c->adapt_tau > 0.0f
                 ? ((c->pct_fp8 + c->pct_mix + c->pct_fp4_max) * v->N + 50) / 100 - c8m
                 : v->n4;
  v->kv4 = v->bs < 64 ? 64 : v->bs;
  const size_t d = c->d, bs = v->bs, N = v->N, BH = (size_t)c->B * c->H;
  v->tile8_qk = bs * d;
  v->tile4_qk = bs * d / 2;
  v->tile8_v = d * bs;
  v->tile4_v = d * v->kv4 / 2;
  v->sf_qk = (d / 64) * 512;
  v->sf_v = (v->kv4 / 64) * 512;
  const size_t n8s = v->n8 > 0 ? v->n8 : 1, n4s = v->n4max > 0 ? v->n4max : 1, nms = v->nm > 0 ? v->nm : 1;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align256(off + bytes);
    if (guards) {
      if (gl && gl->n < kMaxGuards) gl->off[gl->n++] = off;
      off += kGuardBytes;
    }
    return o;
  };
  v->q8 = take(BH * N * v->tile8_qk);
  v->k8 = take(BH * N * v->tile8_qk);
  v->v8 = take(BH * N * v->tile8_v);
  v->q4 = take(BH * N * v->tile4_qk);
  v->k4 = take(BH * N * v->tile4_qk);
  v->v4 = take(BH * N * v->tile4_v);
  v->sfq4 = take(BH * N * v->sf_qk);
  v->sfk4 = take(BH * N * v->sf_qk);
  v->sfv4 = take(BH * N * v->sf_v);
  v->sq = take(BH * N * 4);
  v->sk = take(BH * N * 4);
  v->sv = take(BH * d * 4);
  v->vamax = take(BH * d * 4);
  v->qavg = take(BH * N * d * 4);
  v->qmax = take(BH * N * d * 4);
  v->kavg = take(BH * N * d * 4);
  v->kmax = take(BH * N * d * 4);
  v->tags = take(BH * N * N);
  v->list8 = take(BH * N * n8s * 2);
  v->list4 = take(BH * N * n4s * 2);
  v->listm = take(BH * N * nms * 2);
  v->scores = take((c->flags & DA2_FLAG_EXPORT_SCORES) ? BH * N * N * 4 : 0);
  v->np = (int)((N + 3) / 4 * 4);
  v->dlog = take(N <= 1024 ? BH * N * 2 * (size_t)v->np * 4 : 0);
  v->qt = take(N <= 1024 ? split_region_bytes((int)BH, (int)N, (int)d) : 0);
  v->kt = take(N <= 1024 ? split_region_bytes((int)BH, (int)N, (int)d) : 0);
  v->err = take(4);
  v->total = off;
}

Geo make_geo(const da2_config* c, const da2_views& v) {
  Geo g;
  g.B = c->B; g.H = c->H; g.d = c->d; g.F = c->F; g.Hf = c->Hf; g.Wf = c->Wf;
  g.ph = c->ph; g.pw = c->pw; g.ny = v.ny; g.nx = v.nx; g.N = v.N; g.bs = v.bs;
  g.T = v.T; g.Tp = v.Tp; g.n8 = v.n8; g.n4 = v.n4; g.kv4 = v.kv4; g.nm = v.nm;
  g.n4max = v.n4max;
  g.tau = c->adapt_tau;
  g.sm_scale = c->sm_scale > 0.0f ? c->sm_scale : 1.0f / std::sqrt((float)c->d);
  g.flags = c->flags;
  g.bthd = (c->flags & DA2_FLAG_LAYOUT_BTHD) ? 1 : 0;
  // nothing legitimately waits near 2 s; the test hook shortens the limit to 50 ms
  g.wait_ns = (c->flags & DA2_FLAG_TEST_STALL) ? 50000000ull : 2000000000ull;
  return g;
}

Ws make_ws(void* base, const da2_views& v) {
  uint8_t* b = static_cast<uint8_t*>(base);
  Ws w;
  w.q8 = b + v.q8; w.k8 = b + v.k8; w.v8 = b + v.v8;
  w.q4 = b + v.q4; w.k4 = b + v.k4; w.v4 = b + v.v4;
  w.sfq4 = b + v.sfq4; w.sfk4 = b + v.sfk4; w.sfv4 = b + v.sfv4;
  w.sq = reinterpret_cast<float*>(b + v.sq);
  w.sk = reinterpret_cast<float*>(b + v.sk);
  w.sv = reinterpret_cast<float*>(b + v.sv);
  w.vamax = reinterpret_cast<float*>(b + v.vamax);
  w.qavg = reinterpret_cast<float*>(b + v.qavg);
  w.qmax = reinterpret_cast<float*>(b + v.qmax);
  w.kavg = reinterpret_cast<float*>(b + v.kavg);
  w.kmax = reinterpret_cast<float*>(b + v.kmax);
  w.scores = reinterpret_cast<float*>(b + v.scores);
  w.tags = b + v.tags;
  w.list8 = reinterpret_cast<int16_t*>(b + v.list8);
  w.list4 = reinterpret_cast<int16_t*>(b + v.list4);
  w.listm = reinterpret_cast<int16_t*>(b + v.listm);
  w.err = reinterpret_cast<uint32_t*>(b + v.err);
  w.tile8_qk = v.tile8_qk; w.tile4_qk = v.tile4_qk; w.tile8_v = v.tile8_v; w.tile4_v = v.tile4_v;
  w.sf_qk = v.sf_qk; w.sf_v = v.sf_v;
  w.n8s = v.n8 > 0 ? v.n8 : 1;
  w.n4s = v.n4max > 0 ? v.n4max : 1;
  w.nms = v.nm > 0 ? v.nm : 1;
  return w;
}

// Common checks for the stage calls; fills views / geo / ws on success.
da2_status setup(const da2_config* cfg, void* ws, size_t ws_bytes, da2_views* v, Geo* g, Ws* w,
                 GuardList* gl = nullptr) {
  da2_status s = check_config(cfg);
  if (s != DA2_OK) return s;
  if (!ws) return DA2_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0) return DA2_ERR_ALIGNMENT;
  fill_views(cfg, v, gl);
  if (ws_bytes < v->total) return DA2_ERR_WORKSPACE;
  *g = make_geo(cfg, *v);
  *w = make_ws(ws, *v);
  return DA2_OK;
}

// CUDA error of the calling thread's last failed library call (the launch's own
// cudaGetLastError has consumed it by the time the caller could ask the runtime).
thread_local cudaError_t g_last_cuda = cudaSuccess;

da2_status cuda_status(cudaError_t e) {
  if (e == cudaSuccess) return DA2_OK;
  g_last_cuda = e;
  return DA2_ERR_CUDA;
}

// An NVTX range around one library call (visible in a profiler's timeline; no cost without
// an attached tool).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

// End of a stage call: with DA2_FLAG_DEBUG_CANARY the guard regions are checked (a change
// sets kErrCanary in the error word); a DA2_DEBUG build then waits for the stream and
// returns DA2_ERR_TIMEOUT at once if the error word is set (the word stays set for
// da2_get_error).
da2_status finish_stage(const da2_config* cfg, const Ws& w, void* ws, const GuardList& gl,
                        cudaError_t e, cudaStream_t stream) {
  if (e == cudaSuccess && (cfg->flags & DA2_FLAG_DEBUG_CANARY))
    e = launch_guards(static_cast<uint8_t*>(ws), gl, true, w.err, stream);
#ifdef DA2_DEBUG
  uint32_t h = 0;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&h, w.err, 4, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e == cudaSuccess && h != 0) return DA2_ERR_TIMEOUT;
#endif
  return cuda_status(e);
}

}  // namespace

extern "C" {

da2_status da2_workspace_size(const da2_config* cfg, size_t* bytes) {
  const da2_status s = check_config(cfg);
  if (s != DA2_OK) return s;
  if (!bytes) return DA2_ERR_INVALID_ARG;
  da2_views v;
  fill_views(cfg, &v);
  *bytes = v.total;
  return DA2_OK;
}

da2_status da2_workspace_views(const da2_config* cfg, da2_views* views) {
  const da2_status s = check_config(cfg);
  if (s != DA2_OK) return s;
  if (!views) return DA2_ERR_INVALID_ARG;
  fill_views(cfg, views);
  return DA2_OK;
}

da2_status da2_prepare(const da2_config* cfg, const void* q, const void* k, const void* v,
                       void* ws, size_t ws_bytes, cudaStream_t stream) {
  const NvtxRange range("da2_prepare");
  da2_views vw; Geo g; Ws w; GuardList gl;
  const da2_status s = setup(cfg, ws, ws_bytes, &vw, &g, &w, &gl);
  if (s != DA2_OK) return s;
  if (!q || !k || !v) return DA2_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v)) return DA2_ERR_ALIGNMENT;
  cudaError_t e = cudaSuccess;
  if (cfg->flags & DA2_FLAG_DEBUG_CANARY) e = launch_guards(static_cast<uint8_t*>(ws), gl, false, w.err, stream);
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint8_t* qt = g.N <= 1024 ? base + vw.qt : nullptr;
  uint8_t* kt = g.N <= 1024 ? base + vw.kt : nullptr;
  if (e == cudaSuccess) e = launch_prepare(g, w, q, k, v, qt, kt, stream);
  return finish_stage(cfg, w, ws, gl, e, stream);
}

da2_status da2_draft_select(const da2_config* cfg, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const NvtxRange range("da2_draft_select");
  da2_views vw; Geo g; Ws w; GuardList gl;
  const da2_status s = setup(cfg, ws, ws_bytes, &vw, &g, &w, &gl);
  if (s != DA2_OK) return s;
  uint8_t* base = static_cast<uint8_t*>(ws);
  float* dlog = reinterpret_cast<float*>(base + vw.dlog);
  cudaError_t e = launch_draft_select(g, w, base + vw.qt, base + vw.kt, dlog, vw.np, stream);
#ifdef DA2_DEBUG
  if (e == cudaSuccess) e = launch_check_lists(g, w, stream);
#endif
  return finish_stage(cfg, w, ws, gl, e, stream);
}

da2_status da2_attention(const da2_config* cfg, void* ws, size_t ws_bytes, void* out,
                         cudaStream_t stream) {
  const NvtxRange range("da2_attention");
  da2_views vw; Geo g; Ws w; GuardList gl;
  const da2_status s = setup(cfg, ws, ws_bytes, &vw, &g, &w, &gl);
  if (s != DA2_OK) return s;
  if (!out) return DA2_ERR_INVALID_ARG;
  if (!aligned16(out)) return DA2_ERR_ALIGNMENT;
  return finish_stage(cfg, w, ws, gl, launch_attention_tc(g, w, out, stream), stream);
}

da2_status da2_check_selection(const da2_config* cfg, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const NvtxRange range("da2_check_selection");
  da2_views vw; Geo g; Ws w;
  const da2_status s = setup(cfg, ws, ws_bytes, &vw, &g, &w);
  if (s != DA2_OK) return s;
  return cuda_status(launch_check_lists(g, w, stream));
}

da2_status da2_forward(const da2_config* cfg, const void* q, const void* k, const void* v,
                       void* out, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const NvtxRange range("da2_forward");
  da2_status s = da2_prepare(cfg, q, k, v, ws, ws_bytes, stream);
  if (s != DA2_OK) return s;
  s = da2_draft_select(cfg, ws, ws_bytes, stream);
  if (s != DA2_OK) return s;
  return da2_attention(cfg, ws, ws_bytes, out, stream);
}

namespace {

// The whole path on one stream: copies in, three stages, copy out.
da2_status forward_host_serial(const da2_config* cfg, const void* q_host, const void* k_host,
                               const void* v_host, void* out_host, void* dq, void* dk, void* dv,
                               void* dout, void* ws, size_t ws_bytes, cudaStream_t stream, size_t bytes) {
  cudaError_t e = cudaMemcpyAsync(dq, q_host, bytes, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dk, k_host, bytes, cudaMemcpyHostToDevice, stream);
  if (e == cudaSuccess) e = cudaMemcpyAsync(dv, v_host, bytes, cudaMemcpyHostToDevice, stream);
  if (e != cudaSuccess) return cuda_status(e);
  const da2_status s = da2_forward(cfg, dq, dk, dv, dout, ws, ws_bytes, stream);
  if (s != DA2_OK) return s;
  e = cudaMemcpyAsync(out_host, dout, bytes, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  return cuda_status(e);
}

constexpr int kHostGroups = 16;   // head groups the host-buffer path pipelines over

}  // namespace

// Heads are independent, so the host-buffer path runs as a pipeline over groups of heads:
// the copies in of group g+1 and the copy out of group g-1 overlap the three stages of
// group g (one stream each for copies in, compute and copies out; two sub-workspaces of
// the caller's workspace used alternately). Every stage runs exactly as in da2_forward on
// a configuration of that group's heads.
da2_status da2_forward_host(const da2_config* cfg, const void* q_host, const void* k_host,
                            const void* v_host, void* out_host, void* dq, void* dk, void* dv,
                            void* dout, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const NvtxRange range("da2_forward_host");
  const da2_status s0 = check_config(cfg);
  if (s0 != DA2_OK) return s0;
  if (!q_host || !k_host || !v_host || !out_host || !dq || !dk || !dv || !dout)
    return DA2_ERR_INVALID_ARG;
  const size_t head_bytes = (size_t)cfg->F * cfg->Hf * cfg->Wf * cfg->d * 2;
  const int BH = cfg->B * cfg->H;
  const size_t bytes = head_bytes * BH;
  size_t full_ws = 0;
  if (da2_workspace_size(cfg, &full_ws) != DA2_OK || ws_bytes < full_ws) return DA2_ERR_WORKSPACE;

  // group size: kHostGroups groups when there are enough heads and the two sub-workspaces
  // (plus one error word per group) fit in the caller's workspace
  const int hg = (BH + kHostGroups - 1) / kHostGroups;
  const int G = (BH + hg - 1) / hg;
  da2_config sub = *cfg;
  sub.B = 1;
  sub.H = hg;
  size_t sub_ws = 0;
  if (G < 2 || (cfg->flags & DA2_FLAG_LAYOUT_BTHD) || da2_workspace_size(&sub, &sub_ws) != DA2_OK)
    return forward_host_serial(cfg, q_host, k_host, v_host, out_host, dq, dk, dv, dout, ws, ws_bytes, stream, bytes);
  sub_ws = (sub_ws + 255) & ~size_t(255);
  if (2 * sub_ws + 4 * (size_t)G > ws_bytes)
    return forward_host_serial(cfg, q_host, k_host, v_host, out_host, dq, dk, dv, dout, ws, ws_bytes, stream, bytes);
  uint8_t* ws8 = static_cast<uint8_t*>(ws);
  uint32_t* err_acc = reinterpret_cast<uint32_t*>(ws8 + 2 * sub_ws);   // one word per group

  cudaStream_t st_in = nullptr, st_cmp = nullptr, st_out = nullptr;
  cudaEvent_t ev_start = nullptr, ev_in[kHostGroups] = {}, ev_cmp[kHostGroups] = {}, ev_end[3] = {};
  da2_status status = DA2_OK;
  cudaError_t e = cudaStreamCreateWithFlags(&st_in, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&st_cmp, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&st_out, cudaStreamNonBlocking);
  if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_start, cudaEventDisableTiming);
  for (int g = 0; g < G && e == cudaSuccess; ++g) {
    e = cudaEventCreateWithFlags(&ev_in[g], cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&ev_cmp[g], cudaEventDisableTiming);
  }
  for (int i = 0; i < 3 && e == cudaSuccess; ++i) e = cudaEventCreateWithFlags(&ev_end[i], cudaEventDisableTiming);
  // everything queued on the caller's stream so far comes first
  if (e == cudaSuccess) e = cudaEventRecord(ev_start, stream);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st_in, ev_start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st_cmp, ev_start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st_out, ev_start, 0);
  for (int g = 0; g < G && e == cudaSuccess && status == DA2_OK; ++g) {
    const int h0 = g * hg, nh = BH - h0 < hg ? BH - h0 : hg;
    sub.H = nh;
    const size_t off = head_bytes * h0, len = head_bytes * nh;
    uint8_t* wsg = ws8 + (g & 1) * sub_ws;
    e = cudaMemcpyAsync(static_cast<uint8_t*>(dq) + off, static_cast<const uint8_t*>(q_host) + off, len,
                        cudaMemcpyHostToDevice, st_in);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<uint8_t*>(dk) + off, static_cast<const uint8_t*>(k_host) + off, len,
                          cudaMemcpyHostToDevice, st_in);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<uint8_t*>(dv) + off, static_cast<const uint8_t*>(v_host) + off, len,
                          cudaMemcpyHostToDevice, st_in);
    if (e == cudaSuccess) e = cudaEventRecord(ev_in[g], st_in);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st_cmp, ev_in[g], 0);
    if (e != cudaSuccess) break;
    status = da2_forward(&sub, static_cast<uint8_t*>(dq) + off, static_cast<uint8_t*>(dk) + off,
                         static_cast<uint8_t*>(dv) + off, static_cast<uint8_t*>(dout) + off, wsg, sub_ws, st_cmp);
    if (status != DA2_OK) break;
    // keep this group's error word before the sub-workspace is reused two groups later
    da2_views vw;
    da2_workspace_views(&sub, &vw);
    e = cudaMemcpyAsync(err_acc + g, wsg + vw.err, 4, cudaMemcpyDeviceToDevice, st_cmp);
    if (e == cudaSuccess) e = cudaEventRecord(ev_cmp[g], st_cmp);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(st_out, ev_cmp[g], 0);
    if (e == cudaSuccess)
      e = cudaMemcpyAsync(static_cast<uint8_t*>(out_host) + off, static_cast<const uint8_t*>(dout) + off, len,
                          cudaMemcpyDeviceToHost, st_out);
  }
  // the caller's stream continues after all three
  cudaError_t e2 = cudaSuccess;
  cudaStream_t sts[3] = {st_in, st_cmp, st_out};
  for (int i = 0; i < 3; ++i)
    if (sts[i] && ev_end[i]) {
      if (cudaEventRecord(ev_end[i], sts[i]) == cudaSuccess) cudaStreamWaitEvent(stream, ev_end[i], 0);
    }
  e2 = cudaStreamSynchronize(stream);
  // fold the groups' error words into the error word of the workspace laid out for cfg
  if (e == cudaSuccess && e2 == cudaSuccess && status == DA2_OK) {
    uint32_t words[kHostGroups] = {};
    e2 = cudaMemcpy(words, err_acc, 4 * (size_t)G, cudaMemcpyDeviceToHost);
    uint32_t any = 0;
    for (int g = 0; g < G; ++g) any |= words[g];
    da2_views vfull;
    da2_workspace_views(cfg, &vfull);
    if (e2 == cudaSuccess) e2 = cudaMemcpy(ws8 + vfull.err, &any, 4, cudaMemcpyHostToDevice);
  }
  for (int g = 0; g < kHostGroups; ++g) {
    if (ev_in[g]) cudaEventDestroy(ev_in[g]);
    if (ev_cmp[g]) cudaEventDestroy(ev_cmp[g]);
  }
  for (int i = 0; i < 3; ++i)
    if (ev_end[i]) cudaEventDestroy(ev_end[i]);
  if (ev_start) cudaEventDestroy(ev_start);
  for (int i = 0; i < 3; ++i)
    if (sts[i]) cudaStreamDestroy(sts[i]);
  if (status != DA2_OK) return status;
  return cuda_status(e != cudaSuccess ? e : e2);
}

da2_status da2_get_error(void* ws, size_t ws_bytes, const da2_config* cfg, cudaStream_t stream,
                         uint32_t* word) {
  if (!ws) {                      // the built-in scratch of da2_forward_noalloc
    const da2_status c = check_config(cfg);
    if (c != DA2_OK) return c;
    const da2_status a = noalloc_scratch(&ws, &ws_bytes);
    if (a != DA2_OK) return a;
  }
  da2_views vw; Geo g; Ws w;
  const da2_status s = setup(cfg, ws, ws_bytes, &vw, &g, &w);
  if (s != DA2_OK) return s;
  if (!word) return DA2_ERR_INVALID_ARG;
  uint32_t h = 0;
  cudaError_t e = cudaMemcpyAsync(&h, w.err, 4, cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaMemsetAsync(w.err, 0, 4, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  if (e != cudaSuccess) return cuda_status(e);
  *word = h;
  return h ? DA2_ERR_TIMEOUT : DA2_OK;
}

int da2_last_cuda_error(void) { return (int)g_last_cuda; }

const char* da2_status_string(da2_status s) {
  switch (s) {
    case DA2_OK: return "ok";
    case DA2_ERR_INVALID_ARG: return "invalid argument";
    case DA2_ERR_UNSUPPORTED: return "unsupported shape";
    case DA2_ERR_ALIGNMENT: return "misaligned pointer";
    case DA2_ERR_WORKSPACE: return "workspace too small";
    case DA2_ERR_CUDA: return "CUDA error";
    case DA2_ERR_TIMEOUT: return "device error word set (bounded wait ran out or bad index)";
    case DA2_ERR_SCRATCH_TOO_SMALL: return "workspace larger than the built-in 64 MiB device scratch";
  }
  return "unknown status";
}

}  // extern "C"
