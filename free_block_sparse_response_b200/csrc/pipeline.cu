// The whole SparsePR call behind one entry point (device tensors), and the same call from
// host buffers with the head groups' copies overlapping their neighbours' compute.  Host
// code only: it sequences the stage calls of api.cu (SparsePR abstract, arXiv 2608.18484:
// partition, route, probe rows, fit, corrected sparse attention) on the caller's streams.
#include <cuda_runtime.h>

#include <array>
#include <map>
#include <mutex>

#include "../../include/sparsepr.h"
#include "common.cuh"

namespace spr {
int api_fail(int code, const char* msg);  // sets the thread's last error (api.cu)
}

namespace {

constexpr size_t kAl = 256;
size_t al(size_t x) { return (x + kAl - 1) / kAl * kAl; }

// The fused probe-first order is built for bf16, d = 128, B = 128.
bool fused_shape(int dtype, int d, int block) { return dtype == SPARSEPR_BF16 && d == 128 && block == 128; }

// Byte offsets of the call's intermediates; the stage workspace comes first, so that its
// status header is the call workspace's first 256 bytes.
struct CallLayout {
  size_t stage, key_perm, key_gsize, query_perm, qblock_size, scores, route, pairs, pidx, pout, psparse, M, beta,
      S, total;
};

bool call_layout(int dtype, int32_t Bt, int32_t H, int32_t N, int32_t d, const sparsepr_params* p, CallLayout* L) {
  if (p == nullptr || (dtype != SPARSEPR_BF16 && dtype != SPARSEPR_F32) || p->n_probe < 1 || p->n_probe > N)
    return false;
  const size_t stage = sparsepr_workspace_size(Bt, H, N, d, p);
  if (stage == 0) return false;
  const size_t heads = static_cast<size_t>(Bt) * H, G = static_cast<size_t>(sparsepr_num_groups(N, p->block));
  // route row capacity: k (uniform budget) or G (global budget, rows padded with -1)
  const size_t k = p->route_budget == SPARSEPR_BUDGET_GLOBAL
                       ? G
                       : static_cast<size_t>(sparsepr_route_k(N, p->block, p->density, p->n_probe));
  const size_t P = static_cast<size_t>(p->n_probe), D = static_cast<size_t>(d);
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = al(off + bytes);
    return at;
  };
  L->stage = take(stage);
  L->key_perm = take(4 * heads * G * p->block);
  L->key_gsize = take(4 * heads * G);
  L->query_perm = take(4 * heads * G * p->block);
  L->qblock_size = take(4 * heads * G);
  L->scores = take(4 * heads * G * G);
  L->route = take(4 * heads * G * k);
  L->pairs = take(8 * heads);
  L->pidx = take(4 * heads * P);
  L->pout = take(4 * heads * P * D);
  L->psparse = take(4 * heads * P * D);
  L->M = take(4 * heads * D * D);
  L->beta = take(4 * heads * D);
  L->S = take(fused_shape(dtype, d, p->block) ? 0 : 4 * heads * static_cast<size_t>(N) * D);
  L->total = off;
  return true;
}

// The first device error of a group is kept in the host call's own status word.
__global__ void status_merge_kernel(const int* __restrict__ src, int* __restrict__ dst) {
  const int s = *src;
  if (s != 0) atomicCAS(dst, 0, s);
}

// Events of the host call, per device, created once (the library allocates no memory).
struct HostEvents {
  std::array<cudaEvent_t, 2> in{}, done{};
  cudaEvent_t fin = nullptr;
};
std::mutex g_ev_mu;
std::map<int, HostEvents> g_events;

cudaError_t host_events(HostEvents** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lk(g_ev_mu);
  auto it = g_events.find(dev);
  if (it == g_events.end()) {
    HostEvents ev;
    for (int b = 0; b < 2; ++b) {
      if ((e = cudaEventCreateWithFlags(&ev.in[b], cudaEventDisableTiming)) != cudaSuccess) return e;
      if ((e = cudaEventCreateWithFlags(&ev.done[b], cudaEventDisableTiming)) != cudaSuccess) return e;
    }
    if ((e = cudaEventCreateWithFlags(&ev.fin, cudaEventDisableTiming)) != cudaSuccess) return e;
    it = g_events.emplace(dev, ev).first;
  }
  *out = &it->second;
  return cudaSuccess;
}

size_t elem_bytes(int dtype) { return dtype == SPARSEPR_BF16 ? 2 : 4; }

// Head groups of the host call: the first about half the size of the others, so that
// only a short copy precedes the first compute; the rest equal (the last one ragged).
struct GroupPlan {
  int first, rest, count, max_heads;
  int start(int g) const { return g == 0 ? 0 : first + (g - 1) * rest; }
};
GroupPlan group_plan(int heads, int groups) {
  GroupPlan gp;
  if (groups <= 1 || heads <= 1) {
    gp.first = gp.rest = gp.max_heads = heads;
    gp.count = 1;
    return gp;
  }
  gp.first = (heads + 2 * groups - 2) / (2 * groups - 1);
  gp.rest = (heads - gp.first + groups - 2) / (groups - 1);
  if (gp.rest < 1) gp.rest = 1;
  gp.count = 1 + (heads - gp.first + gp.rest - 1) / gp.rest;
  gp.max_heads = gp.first > gp.rest ? gp.first : gp.rest;
  return gp;
}

}  // namespace

extern "C" {

size_t sparsepr_call_workspace_size(int dtype, int32_t Bt, int32_t H, int32_t N, int32_t d,
                                    const sparsepr_params* params) {
  CallLayout L;
  return call_layout(dtype, Bt, H, N, d, params, &L) ? L.total : 0;
}

int sparsepr_attention(const void* Q, const void* K, const void* V, int dtype, int32_t Bt, int32_t H, int32_t N,
                       int32_t d, const sparsepr_params* p, void* O, void* ws, sparsepr_stream_t stream) {
  if (!Q || !K || !V || !O || !ws || !p) return spr::api_fail(SPARSEPR_ERR_INVALID_ARG, "null pointer argument");
  CallLayout L;
  if (!call_layout(dtype, Bt, H, N, d, p, &L))
    return spr::api_fail(SPARSEPR_ERR_INVALID_ARG, "invalid sizes or parameters for the call (n_probe must be in [1, N])");
  char* w = static_cast<char*>(ws);
  auto I = [&](size_t off) { return reinterpret_cast<int32_t*>(w + off); };
  auto F = [&](size_t off) { return reinterpret_cast<float*>(w + off); };
  void* sws = w + L.stage;
  int rc;
  if ((rc = sparsepr_partition(Q, K, dtype, Bt, H, N, d, p, nullptr, I(L.key_perm), I(L.key_gsize), I(L.query_perm),
                               I(L.qblock_size), F(L.scores), sws, stream)))
    return rc;
  int32_t k = 0;
  if ((rc = sparsepr_route(F(L.scores), I(L.key_gsize), I(L.qblock_size), Bt, H, N, p, I(L.route), &k,
                           reinterpret_cast<int64_t*>(w + L.pairs), sws, stream)))
    return rc;
  if ((rc = sparsepr_probe_rows(N, p->n_probe, Bt, H, I(L.pidx), stream))) return rc;
  const bool fused = fused_shape(dtype, d, p->block);
  if (!fused && (rc = sparsepr_sparse_attn(Q, K, V, dtype, Bt, H, N, d, p->block, I(L.key_perm), I(L.key_gsize),
                                           I(L.query_perm), I(L.qblock_size), I(L.route), k, p->scale, F(L.S), sws,
                                           stream)))
    return rc;
  if ((rc = sparsepr_probe_dense(Q, K, V, dtype, Bt, H, N, d, p->block, I(L.pidx), p->n_probe, I(L.key_perm),
                                 I(L.key_gsize), I(L.query_perm), I(L.route), k, p->scale, F(L.pout), F(L.psparse),
                                 sws, stream)))
    return rc;
  if ((rc = sparsepr_fit_residual(F(L.psparse), F(L.pout), nullptr, Bt, H, d, p->n_probe, p->ridge_lambda, p->rank,
                                  p->weight_mode, F(L.M), F(L.beta), sws, stream)))
    return rc;
  if (fused)
    return sparsepr_sparse_attn_apply(Q, K, V, dtype, Bt, H, N, d, p->block, I(L.key_perm), I(L.key_gsize),
                                      I(L.query_perm), I(L.qblock_size), I(L.route), k, p->scale, F(L.M), F(L.beta),
                                      I(L.pidx), p->n_probe, F(L.pout), O, sws, stream);
  return sparsepr_apply_residual(F(L.S), F(L.M), F(L.beta), I(L.pidx), F(L.pout), Bt, H, N, d, p->n_probe, O, dtype,
                                 stream);
}

size_t sparsepr_host_workspace_size(int dtype, int32_t Bt, int32_t H, int32_t N, int32_t d,
                                    const sparsepr_params* params, int32_t groups) {
  if (groups < 1 || Bt < 1 || H < 1) return 0;
  const int hg = group_plan(Bt * H, groups).max_heads;
  const size_t call = sparsepr_call_workspace_size(dtype, 1, hg, N, d, params);
  if (call == 0) return 0;
  const size_t tensor = al(static_cast<size_t>(hg) * N * d * elem_bytes(dtype));
  return kAl + al(call) + 2 * 4 * tensor;
}

int sparsepr_attention_host(const void* Q, const void* K, const void* V, int dtype, int32_t Bt, int32_t H,
                            int32_t N, int32_t d, const sparsepr_params* p, void* O, int32_t groups, void* ws,
                            sparsepr_stream_t stream, sparsepr_stream_t copy_stream) {
  if (!Q || !K || !V || !O || !ws || !p) return spr::api_fail(SPARSEPR_ERR_INVALID_ARG, "null pointer argument");
  if (groups < 1) return spr::api_fail(SPARSEPR_ERR_INVALID_ARG, "groups must be >= 1");
  if (stream == copy_stream) return spr::api_fail(SPARSEPR_ERR_INVALID_ARG, "the copy stream must differ from the compute stream");
  if (sparsepr_host_workspace_size(dtype, Bt, H, N, d, p, groups) == 0)
    return spr::api_fail(SPARSEPR_ERR_INVALID_ARG, "invalid sizes or parameters for the call (n_probe must be in [1, N])");
  const int heads = Bt * H;
  const GroupPlan plan = group_plan(heads, groups);
  const int hg = plan.max_heads, ng = plan.count;
  const size_t call = al(sparsepr_call_workspace_size(dtype, 1, hg, N, d, p));
  const size_t per_head = static_cast<size_t>(N) * d * elem_bytes(dtype);
  const size_t tensor = al(static_cast<size_t>(hg) * per_head);
  char* base = static_cast<char*>(ws);
  int* agg = reinterpret_cast<int*>(base);  // this call's status word (sparsepr_check reads it)
  char* cws = base + kAl;
  char* stg = cws + call;
  auto dbuf = [&](int b, int t) { return stg + (static_cast<size_t>(b) * 4 + t) * tensor; };
  const char* hq = static_cast<const char*>(Q);
  const char* hk = static_cast<const char*>(K);
  const char* hv = static_cast<const char*>(V);
  char* ho = static_cast<char*>(O);
  cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream), xs = reinterpret_cast<cudaStream_t>(copy_stream);
  HostEvents* ev = nullptr;
  cudaError_t e = host_events(&ev);
  if (e != cudaSuccess) return spr::api_fail(SPARSEPR_ERR_CUDA, cudaGetErrorString(e));
  auto cuda_err = [&](cudaError_t err) { return spr::api_fail(SPARSEPR_ERR_CUDA, cudaGetErrorString(err)); };
  if ((e = cudaMemsetAsync(agg, 0, sizeof(int), cs)) != cudaSuccess) return cuda_err(e);
  // the copy stream starts after whatever the compute stream holds (the status reset)
  if ((e = cudaEventRecord(ev->fin, cs)) != cudaSuccess || (e = cudaStreamWaitEvent(xs, ev->fin, 0)) != cudaSuccess)
    return cuda_err(e);
  // copy order: in(0), in(1), [done 0] out(0), in(2), [done 1] out(1), in(3), ... so that
  // group g + 1 lands during group g, and a buffer is refilled only after its last
  // group's output has been copied back
  auto span = [&](int g, int* h0, int* nh) {
    *h0 = plan.start(g);
    const int want = g == 0 ? plan.first : plan.rest;
    *nh = heads - *h0 < want ? heads - *h0 : want;
  };
  auto copy_in = [&](int g) -> cudaError_t {
    int h0, nh;
    span(g, &h0, &nh);
    const int b = g & 1;
    const size_t off = static_cast<size_t>(h0) * per_head, bytes = static_cast<size_t>(nh) * per_head;
    cudaError_t r;
    if ((r = cudaMemcpyAsync(dbuf(b, 0), hq + off, bytes, cudaMemcpyHostToDevice, xs)) != cudaSuccess) return r;
    if ((r = cudaMemcpyAsync(dbuf(b, 1), hk + off, bytes, cudaMemcpyHostToDevice, xs)) != cudaSuccess) return r;
    if ((r = cudaMemcpyAsync(dbuf(b, 2), hv + off, bytes, cudaMemcpyHostToDevice, xs)) != cudaSuccess) return r;
    return cudaEventRecord(ev->in[b], xs);
  };
  if ((e = copy_in(0)) != cudaSuccess) return cuda_err(e);
  for (int g = 0; g < ng; ++g) {
    int h0, nh;
    span(g, &h0, &nh);
    const int b = g & 1;
    if (g + 1 < ng && (e = copy_in(g + 1)) != cudaSuccess) return cuda_err(e);
    if ((e = cudaStreamWaitEvent(cs, ev->in[b], 0)) != cudaSuccess) return cuda_err(e);
    const int rc = sparsepr_attention(dbuf(b, 0), dbuf(b, 1), dbuf(b, 2), dtype, 1, nh, N, d, p, dbuf(b, 3), cws,
                                      stream);
    if (rc != SPARSEPR_OK) return rc;
    status_merge_kernel<<<1, 1, 0, cs>>>(reinterpret_cast<const int*>(cws + 0), agg);  // header status: first word
    if ((e = cudaGetLastError()) != cudaSuccess) return cuda_err(e);
    spr::note_launches(1);
    if ((e = cudaEventRecord(ev->done[b], cs)) != cudaSuccess || (e = cudaStreamWaitEvent(xs, ev->done[b], 0)) != cudaSuccess)
      return cuda_err(e);
    const size_t off = static_cast<size_t>(h0) * per_head, bytes = static_cast<size_t>(nh) * per_head;
    if ((e = cudaMemcpyAsync(ho + off, dbuf(b, 3), bytes, cudaMemcpyDeviceToHost, xs)) != cudaSuccess)
      return cuda_err(e);
  }
  // the host O is complete once the compute stream is
  if ((e = cudaEventRecord(ev->fin, xs)) != cudaSuccess || (e = cudaStreamWaitEvent(cs, ev->fin, 0)) != cudaSuccess)
    return cuda_err(e);
  return SPARSEPR_OK;
}

}  // extern "C"
