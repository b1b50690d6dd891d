// extern "C" entry points of libsparsepr (see include/sparsepr.h for the contract).
#include <cmath>
#include <algorithm>
#include <cstdarg>
#include <cstdio>
#include <atomic>
#include <cstring>
#include <initializer_list>
#include <mutex>
#include <string>

#include "../../include/sparsepr.h"

#include <initializer_list>
#include "attention.cuh"
#include "common.cuh"
#include "fit.cuh"
#include "partition.cuh"
#include "route.cuh"

namespace spr {
namespace {
std::atomic<unsigned long long> g_launches{0};
}
void note_launches(int n) { g_launches.fetch_add(static_cast<unsigned long long>(n), std::memory_order_relaxed); }
}  // namespace spr

namespace {

thread_local std::string g_last_error;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

int cuda_fail(cudaError_t e, const char* where) {
  return fail(SPARSEPR_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

}  // namespace

namespace spr {
int api_fail(int code, const char* msg) { return fail(code, "%s", msg); }
}  // namespace spr

namespace {

// Row stride of the distance matrix: a whole number of 128-byte lines, so that every
// row starts on a line and the distance kernel's 64-byte stores never split a sector.
size_t dmat_ld(int G) { return static_cast<size_t>(G + 31) / 32 * 32; }

// The tensor-core fill's stored tail rows: up to 32K unplaced items (of all heads), each
// row a whole number of 128-group chunks.
int tail_cap(int heads, int N) {
  return static_cast<int>(std::min<long long>(1ll << 15, static_cast<long long>(heads) * N));
}
int tail_ld(int G) { return (G + 127) / 128 * 128; }


#define SPR_CUDA(call, where)                       \
  do {                                              \
    cudaError_t e_ = (call);                        \
    if (e_ != cudaSuccess) return cuda_fail(e_, where); \
  } while (0)

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// Byte offsets of every scratch region inside the caller's workspace.
struct Layout {
  size_t header = 0, sample_idx, gamma, gamma_hi, gamma_lo, nrm, cent_k, cent_q, wf, whi, wlo, eg, dmat,
         prop_g0, prop_v0, labels, room, cnt, offs, cursor, closed, bucket, list0, list1, list_len, prop_g, prop_v,
         perm_tmp, perm_cursor, qblk, partial, fit, kv_grouped, mhilo, ovf, dtail, tailpos, wcomp, openg, total;
};

Layout make_layout(int heads, int N, int d, int block, int S, int P) {
  const size_t H = heads, n = N, G = spr::ceil_div(N, block), D = d;
  Layout L;
  size_t off = align_up(sizeof(spr::WorkspaceHeader));
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off = align_up(off + bytes);
    return at;
  };
  // Regions read by the calls after partition come first, so that their offsets depend
  // only on the shapes (and P) each of those calls knows.  The fit's scratch comes first
  // of all, sized for the largest P it takes: the fit call knows neither N nor the block.
  L.fit = take(sizeof(double) * H * spr::fit_scratch_doubles(spr::fit_max_probes(d), d));
  L.kv_grouped = take(2 * 2 * H * G * block * D);  // K and V in key-group order, bf16
  L.mhilo = take(2 * 2 * H * D * D);                // M as bf16 hi and lo (fused correction)
  L.partial = take(P > 0 ? spr::probe_partial_bytes(heads, P, static_cast<int>(G), d) : 0);
  L.sample_idx = take(sizeof(int) * static_cast<size_t>(S));
  L.gamma = take(sizeof(float) * H * D * D);
  L.gamma_hi = take(2 * H * D * D);
  L.gamma_lo = take(2 * H * D * D);
  L.nrm = take(sizeof(float) * H * n);
  L.cent_k = take(sizeof(float) * H * G * D);
  L.cent_q = take(sizeof(float) * H * G * D);
  L.wf = take(sizeof(float) * H * G * D);
  L.whi = take(2 * H * G * D);
  L.wlo = take(2 * H * G * D);
  L.eg = take(sizeof(float) * H * G);
  L.dmat = take(sizeof(float) * H * n * dmat_ld(G));
  L.prop_g0 = take(sizeof(int) * H * n);
  L.prop_v0 = take(sizeof(float) * H * n);
  L.labels = take(sizeof(int) * H * n);
  L.room = take(sizeof(int) * H * G);
  L.cnt = take(sizeof(int) * H * G);
  L.offs = take(sizeof(int) * H * G);
  L.cursor = take(sizeof(int) * H * G);
  L.closed = take(sizeof(unsigned int) * H * ((G + 31) / 32));
  L.bucket = take(sizeof(unsigned long long) * H * n);
  L.list0 = take(sizeof(int) * H * n);
  L.list1 = take(sizeof(int) * H * n);
  L.list_len = take(sizeof(int) * std::max<size_t>(4, 2 * H));
  L.prop_g = take(sizeof(int) * H * n);
  L.prop_v = take(sizeof(float) * H * n);
  L.perm_tmp = take(sizeof(int) * H * G * block);
  L.perm_cursor = take(sizeof(int) * H * G);
  L.qblk = take(sizeof(int) * H * n);
  L.ovf = take(sizeof(int) * (H * G + 2));
  L.dtail = take(sizeof(float) * tail_cap(heads, N) * tail_ld(static_cast<int>(G)));
  L.tailpos = take(sizeof(int) * H * n);
  L.wcomp = take(2 * 2 * H * G * D);          // the open groups' W, bf16 hi and lo
  L.openg = take(sizeof(int) * (H * G + H));  // packed column -> group, and counts
  L.total = off;
  return L;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

spr::WorkspaceHeader* header(void* ws) { return static_cast<spr::WorkspaceHeader*>(ws); }

int check_shape(int32_t Bt, int32_t H, int32_t N, int32_t d) {
  if (Bt < 1 || H < 1 || N < 1) return fail(SPARSEPR_ERR_INVALID_ARG, "Bt, H and N must be >= 1");
  if (d != 64 && d != 128) return fail(SPARSEPR_ERR_UNSUPPORTED, "head dim %d: only 64 and 128 are built", d);
  if (static_cast<long long>(Bt) * H * N > (1ll << 30))
    return fail(SPARSEPR_ERR_UNSUPPORTED, "Bt*H*N above 2^30 tokens per call");
  return SPARSEPR_OK;
}

int check_block(int32_t block) {
  if (block != 64 && block != 128) return fail(SPARSEPR_ERR_UNSUPPORTED, "block %d: only 64 and 128 are built", block);
  return SPARSEPR_OK;
}

// Q, K, V are read with 16-byte vector and TMA loads.
int check_aligned(std::initializer_list<const void*> ptrs) {
  for (const void* q : ptrs)
    if ((reinterpret_cast<uintptr_t>(q) & 15u) != 0)
      return fail(SPARSEPR_ERR_INVALID_ARG, "Q, K and V must start on 16-byte boundaries");
  return SPARSEPR_OK;
}

int check_dtype(int dtype) {
  if (dtype != SPARSEPR_BF16 && dtype != SPARSEPR_F32) return fail(SPARSEPR_ERR_INVALID_ARG, "unknown dtype %d", dtype);
  return SPARSEPR_OK;
}

static_assert(SPARSEPR_RIDGE_RELATIVE == spr::kRidgeRelative, "ridge flag of the ABI and the kernel");

// Probe weights (SPARSEPR_WEIGHT_*), optionally | SPARSEPR_RIDGE_RELATIVE.
int check_weight_mode(int weight_mode) {
  const int w = weight_mode & ~SPARSEPR_RIDGE_RELATIVE;
  if (w != SPARSEPR_WEIGHT_INV_NORM && w != SPARSEPR_WEIGHT_UNIFORM)
    return fail(SPARSEPR_ERR_INVALID_ARG, "unknown weight_mode %d", weight_mode);
  return SPARSEPR_OK;
}

float resolve_scale(float scale, int d) { return scale > 0.f ? scale : 1.0f / std::sqrt(static_cast<float>(d)); }

constexpr float kLog2e = 1.4426950408889634f;

}  // namespace

extern "C" {

int32_t sparsepr_num_groups(int32_t N, int32_t block) {
  if (N < 1 || block < 1) return 0;
  return spr::ceil_div(N, block);
}

int32_t sparsepr_route_k(int32_t N, int32_t block, double density, int32_t n_probe) {
  if (N < 1 || block < 1) return 0;
  const int32_t G = spr::ceil_div(N, block);
  const double num = density * static_cast<double>(N) * static_cast<double>(N) -
                     static_cast<double>(n_probe) * static_cast<double>(N);
  const double k = std::floor(num / (static_cast<double>(N) * static_cast<double>(block)));
  if (!(k >= 1.0)) return 1;
  if (k >= static_cast<double>(G)) return G;
  return static_cast<int32_t>(k);
}

size_t sparsepr_workspace_size(int32_t Bt, int32_t H, int32_t N, int32_t d, const sparsepr_params* p) {
  if (p == nullptr || check_shape(Bt, H, N, d) != SPARSEPR_OK || check_block(p->block) != SPARSEPR_OK) return 0;
  return make_layout(Bt * H, N, d, p->block, p->n_sampled > 0 ? p->n_sampled : 1, p->n_probe).total;
}

const char* sparsepr_last_error(void) { return g_last_error.c_str(); }

int sparsepr_check(const void* ws, sparsepr_stream_t stream) {
  if (ws == nullptr) return fail(SPARSEPR_ERR_INVALID_ARG, "null workspace");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  SPR_CUDA(cudaStreamSynchronize(st), "sparsepr_check: stream");
  int status = 0;
  SPR_CUDA(cudaMemcpy(&status, ws, sizeof(int), cudaMemcpyDeviceToHost), "sparsepr_check: read status");
  if (status != SPARSEPR_OK) return fail(status, "device-side error %d recorded in the workspace", status);
  return SPARSEPR_OK;
}

int sparsepr_reset_workspace(void* ws, sparsepr_stream_t stream) {
  if (!ws) return fail(SPARSEPR_ERR_INVALID_ARG, "null workspace");
  SPR_CUDA(cudaMemsetAsync(ws, 0, sizeof(spr::WorkspaceHeader), reinterpret_cast<cudaStream_t>(stream)),
           "reset workspace");
  return SPARSEPR_OK;
}

// The partition; `tr` (test-only, may be null) receives copies of its internal state.
static int partition_impl(const void* Q, const void* K, int dtype, int32_t Bt, int32_t H, int32_t N, int32_t d,
                          const sparsepr_params* p, const int32_t* sample_idx, int32_t* key_perm,
                          int32_t* key_gsize, int32_t* query_perm, int32_t* qblock_size, float* block_scores,
                          const sparsepr_partition_trace* tr, void* ws, sparsepr_stream_t stream) {
  int rc;
  if ((rc = check_shape(Bt, H, N, d)) || (rc = check_dtype(dtype))) return rc;
  if (p == nullptr) return fail(SPARSEPR_ERR_INVALID_ARG, "null params");
  if ((rc = check_block(p->block))) return rc;
  if (!Q || !K || !key_perm || !key_gsize || !query_perm || !qblock_size || !block_scores || !ws)
    return fail(SPARSEPR_ERR_INVALID_ARG, "null pointer argument");
  if ((rc = check_aligned({Q, K}))) return rc;
  if (p->n_sampled < 1 || p->n_sampled > N) return fail(SPARSEPR_ERR_INVALID_ARG, "n_sampled must be in [1, N]");
  if (p->kmeans_iters < 0 || p->kmeans_iters > 64) return fail(SPARSEPR_ERR_INVALID_ARG, "kmeans_iters must be in [0, 64]");
  if (spr::ceil_div(N, p->block) > 1024)
    return fail(SPARSEPR_ERR_UNSUPPORTED, "more than 1024 groups per head (N / block) is not built");
  if (p->partition_mode != SPARSEPR_PARTITION_RESPONSE && p->partition_mode != SPARSEPR_PARTITION_SEMANTIC)
    return fail(SPARSEPR_ERR_INVALID_ARG, "unknown partition_mode %d", p->partition_mode);
  const bool semantic = p->partition_mode == SPARSEPR_PARTITION_SEMANTIC;
  if (p->route_scores < SPARSEPR_ROUTE_CENTROID || p->route_scores > SPARSEPR_ROUTE_LSE)
    return fail(SPARSEPR_ERR_INVALID_ARG, "unknown route_scores %d", p->route_scores);
  if (p->route_scores == SPARSEPR_ROUTE_LSE && (dtype == SPARSEPR_F32 || d != 128 || p->block != 128))
    return fail(SPARSEPR_ERR_UNSUPPORTED, "LSE routing scores are built for bf16, d = 128, block = 128");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int heads = Bt * H, B = p->block, G = spr::ceil_div(N, B), S = p->n_sampled;
  const bool f32 = dtype == SPARSEPR_F32;
  const float tau = resolve_scale(p->scale, d);
  const Layout L = make_layout(heads, N, d, B, S, p->n_probe);
  spr::WorkspaceHeader* hdr = header(ws);
  int* status = &hdr->status;
  SPR_CUDA(cudaMemsetAsync(ws, 0, sizeof(spr::WorkspaceHeader), st), "partition: reset status");
  const int* sidx = sample_idx;
  if (sidx == nullptr) {
    SPR_CUDA(spr::launch_midpoint_stride(at<int>(ws, L.sample_idx), N, S, st), "partition: sample");
    sidx = at<int>(ws, L.sample_idx);
  }
  // test-only copies of the internal state (nothing below reads them)
  auto copy_out = [&](void* dst, const void* src, size_t bytes, const char* what) -> int {
    if (dst != nullptr) SPR_CUDA(cudaMemcpyAsync(dst, src, bytes, cudaMemcpyDeviceToDevice, st), what);
    return SPARSEPR_OK;
  };
  if (tr && (rc = copy_out(tr->sample_idx, sidx, sizeof(int) * S, "trace: sample"))) return rc;
  float* gamma = at<float>(ws, L.gamma);
  __nv_bfloat16* ghi = at<__nv_bfloat16>(ws, L.gamma_hi);
  __nv_bfloat16* glo = at<__nv_bfloat16>(ws, L.gamma_lo);
  float* nrm = at<float>(ws, L.nrm);
  float* wf = at<float>(ws, L.wf);
  __nv_bfloat16* whi = at<__nv_bfloat16>(ws, L.whi);
  __nv_bfloat16* wlo = at<__nv_bfloat16>(ws, L.wlo);
  float* eg = at<float>(ws, L.eg);

  float* dmat = at<float>(ws, L.dmat);
  spr::FillArgs fa{};
  fa.D = dmat;
  fa.ldd = dmat_ld(G);
  fa.prop_g0 = at<int>(ws, L.prop_g0);
  fa.prop_v0 = at<float>(ws, L.prop_v0);
  // bf16, d = 128: the tensor-core assignment kernel (distances and fill in one launch)
  const bool tc_assign = !f32 && d == 128;
  fa.heads = heads;
  fa.n = N;
  fa.G = G;
  fa.cap = B;
  fa.labels = at<int>(ws, L.labels);
  fa.room = at<int>(ws, L.room);
  fa.cnt = at<int>(ws, L.cnt);
  fa.offs = at<int>(ws, L.offs);
  fa.cursor = at<int>(ws, L.cursor);
  fa.closed = at<unsigned int>(ws, L.closed);
  fa.bucket = at<unsigned long long>(ws, L.bucket);
  fa.list0 = at<int>(ws, L.list0);
  fa.list1 = at<int>(ws, L.list1);
  fa.list_len = at<int>(ws, L.list_len);
  fa.prop_g = at<int>(ws, L.prop_g);
  fa.prop_v = at<float>(ws, L.prop_v);
  fa.hdr = hdr;

  // One side of the partition: balanced k-means of the rows of X under metric gamma.
  auto cluster = [&](const void* X, float* cent, int32_t* perm, int32_t* sizes, float* tr_dist,
                     int32_t* tr_labels) -> int {
    spr::RowGemmArgs ra{};
    ra.X = X;
    ra.f32 = f32;
    ra.heads = heads;
    ra.n = N;
    ra.d = d;
    ra.status = status;
    if (!f32) SPR_CUDA(spr::launch_split_bf16(gamma, ghi, glo, static_cast<size_t>(heads) * d * d, st), "split gamma");
    ra.ncols = d;
    ra.Bhi = ghi;
    ra.Blo = glo;
    ra.Bf32 = gamma;
    ra.nrm_out = nrm;
    if (tc_assign)
      SPR_CUDA(spr::launch_row_norms_tc(static_cast<const __nv_bfloat16*>(X), ghi, glo, heads, N, nrm, hdr, st),
               "row norms");
    else
      SPR_CUDA(spr::launch_rowgemm(ra, false, st), "row norms");
    SPR_CUDA(spr::launch_chunk_perm(perm, sizes, N, G, B, heads, st), "chunk start");
    SPR_CUDA(spr::launch_centroid(X, f32, N, perm, sizes, G, B, heads, d, cent, st), "centroids");
    if (p->kmeans_iters > 0)
      SPR_CUDA(spr::launch_wmat(cent, gamma, G, heads, d, wf, whi, wlo, eg, st), "gamma centroids");
    int* members = at<int>(ws, L.perm_tmp);
    int* msize = at<int>(ws, L.perm_cursor);
    for (int t = 0; t < p->kmeans_iters; ++t) {
      ra.ncols = G;
      ra.Bhi = whi;
      ra.Blo = wlo;
      ra.Bf32 = wf;
      ra.nrm = nrm;
      ra.ecol = eg;
      ra.tau2 = semantic ? 1.0f : tau * tau;  // raw squared distances for the semantic rule
      ra.Dout = dmat;
      ra.ldd = fa.ldd;
      ra.prop_g = at<int>(ws, L.prop_g0);
      ra.prop_v = at<float>(ws, L.prop_v0);
      ra.nrm_out = nullptr;
      if (tc_assign) {
        // bf16, d = 128: proposals and fill in one tensor-core kernel, no distance matrix
        // (the parity trace has it store the first round's rows)
        spr::AssignArgs aa{};
        aa.heads = heads;
        aa.n = N;
        aa.G = G;
        aa.cap = B;
        aa.tau2 = ra.tau2;
        aa.nrm = nrm;
        aa.ecol = eg;
        aa.labels = fa.labels;
        aa.room = fa.room;
        aa.cnt = fa.cnt;
        aa.offs = fa.offs;
        aa.cursor = fa.cursor;
        aa.closed = fa.closed;
        aa.bucket = fa.bucket;
        aa.list[0] = fa.list0;
        aa.list[1] = fa.list1;
        aa.list_len = fa.list_len;
        aa.prop_g = fa.prop_g;
        aa.prop_v = fa.prop_v;
        aa.members = members;
        aa.msize = msize;
        aa.ovf_list = at<int>(ws, L.ovf);
        aa.ovf_total = at<int>(ws, L.ovf) + static_cast<size_t>(heads) * G;
        aa.Dout = tr_dist != nullptr ? dmat : nullptr;
        aa.Dtail = at<float>(ws, L.dtail);
        aa.ldt = tail_ld(G);
        aa.tail_cap = tail_cap(heads, N);
        aa.tailpos = at<int>(ws, L.tailpos);
        aa.wc_hi = at<__nv_bfloat16>(ws, L.wcomp);
        aa.wc_lo = aa.wc_hi + static_cast<size_t>(heads) * G * d;
        aa.open_g = at<int>(ws, L.openg);
        aa.n_open = aa.open_g + static_cast<size_t>(heads) * G;
        aa.ldd = static_cast<int>(fa.ldd);
        aa.hdr = hdr;
        SPR_CUDA(spr::launch_assign_tc(static_cast<const __nv_bfloat16*>(X), whi, wlo, aa, st), "assignment");
      } else {
        SPR_CUDA(spr::launch_rowgemm(ra, true, st), "distances");
      }
      if (tr_dist != nullptr)
        SPR_CUDA(cudaMemcpy2DAsync(tr_dist + static_cast<size_t>(t) * heads * N * G, sizeof(float) * G, dmat,
                                   sizeof(float) * fa.ldd, sizeof(float) * G, static_cast<size_t>(heads) * N,
                                   cudaMemcpyDeviceToDevice, st),
                 "trace: distances");
      if (!tc_assign) SPR_CUDA(spr::launch_fill(fa, st), "capacity fill");
      if (tr_labels != nullptr &&
          (rc = copy_out(tr_labels + static_cast<size_t>(t) * heads * N, fa.labels, sizeof(int) * heads * N,
                         "trace: labels")))
        return rc;
      // members (kept by the tensor-core fill, else scattered from the labels) -> sorted
      // permutation, the new means and the next iteration's W and e
      if (!tc_assign)
        SPR_CUDA(spr::launch_perm_scatter(fa.labels, N, G, B, heads, msize, members, status, st), "members");
      SPR_CUDA(spr::launch_group_update(X, f32, N, msize, members, G, B, heads, d, gamma, perm, sizes, cent, wf, whi,
                                        wlo, eg, st),
               "group update");
    }
    return SPARSEPR_OK;
  };

  float* cent_k = at<float>(ws, L.cent_k);
  float* cent_q = at<float>(ws, L.cent_q);
  // keys: profiles against the sampled queries -> gamma = Q_S^T Q_S (semantic: identity)
  const size_t gamma_bytes = sizeof(float) * heads * d * d, cent_bytes = sizeof(float) * heads * G * d;
  if (semantic) SPR_CUDA(spr::launch_identity(gamma, heads, d, st), "identity metric");
  else SPR_CUDA(spr::launch_gram(Q, f32, static_cast<size_t>(N) * d, sidx, S, heads, d, gamma, st), "Q_S gram");
  if (tr && (rc = copy_out(tr->key_gamma, gamma, gamma_bytes, "trace: key metric"))) return rc;
  if ((rc = cluster(K, cent_k, key_perm, key_gsize, tr ? tr->key_dist : nullptr, tr ? tr->key_labels : nullptr)))
    return rc;
  if (tr && (rc = copy_out(tr->mu, cent_k, cent_bytes, "trace: mu"))) return rc;
  // queries: coordinates against the key-group mean keys -> gamma = mu^T mu (semantic:
  // the raw queries, identity)
  if (semantic) SPR_CUDA(spr::launch_identity(gamma, heads, d, st), "identity metric");
  else SPR_CUDA(spr::launch_gram(cent_k, true, static_cast<size_t>(G) * d, nullptr, G, heads, d, gamma, st), "mu gram");
  if (tr && (rc = copy_out(tr->query_gamma, gamma, gamma_bytes, "trace: query metric"))) return rc;
  if ((rc = cluster(Q, cent_q, query_perm, qblock_size, tr ? tr->query_dist : nullptr,
                    tr ? tr->query_labels : nullptr)))
    return rc;
  if (tr && (rc = copy_out(tr->qbar, cent_q, cent_bytes, "trace: qbar"))) return rc;
  SPR_CUDA(spr::launch_block_scores(cent_q, cent_k, G, heads, d, tau, block_scores, st), "block scores");
  SPR_CUDA(spr::launch_route_scores(p->route_scores, block_scores, K, N, heads, G, G, key_perm, key_gsize, cent_q, tau,
                                    st),
           "routing scores");
  return SPARSEPR_OK;
}

int sparsepr_partition(const void* Q, const void* K, int dtype, int32_t Bt, int32_t H, int32_t N, int32_t d,
                       const sparsepr_params* p, const int32_t* sample_idx, int32_t* key_perm,
                       int32_t* key_gsize, int32_t* query_perm, int32_t* qblock_size, float* block_scores,
                       void* ws, sparsepr_stream_t stream) {
  return partition_impl(Q, K, dtype, Bt, H, N, d, p, sample_idx, key_perm, key_gsize, query_perm, qblock_size,
                        block_scores, nullptr, ws, stream);
}

int sparsepr_test_partition_trace(const void* Q, const void* K, int dtype, int32_t Bt, int32_t H, int32_t N,
                                  int32_t d, const sparsepr_params* p, const int32_t* sample_idx, int32_t* key_perm,
                                  int32_t* key_gsize, int32_t* query_perm, int32_t* qblock_size,
                                  float* block_scores, const sparsepr_partition_trace* trace, void* ws,
                                  sparsepr_stream_t stream) {
  if (trace == nullptr) return fail(SPARSEPR_ERR_INVALID_ARG, "null trace");
  return partition_impl(Q, K, dtype, Bt, H, N, d, p, sample_idx, key_perm, key_gsize, query_perm, qblock_size,
                        block_scores, trace, ws, stream);
}

int sparsepr_route(const float* block_scores, const int32_t* key_gsize, const int32_t* qblock_size, int32_t Bt,
                   int32_t H, int32_t N, const sparsepr_params* p, int32_t* route, int32_t* k_out,
                   int64_t* executed_pairs, void* ws, sparsepr_stream_t stream) {
  int rc;
  if ((rc = check_shape(Bt, H, N, 64))) return rc;
  if (p == nullptr) return fail(SPARSEPR_ERR_INVALID_ARG, "null params");
  if ((rc = check_block(p->block))) return rc;
  if (!block_scores || !key_gsize || !qblock_size || !route || !ws)
    return fail(SPARSEPR_ERR_INVALID_ARG, "null pointer argument");
  if (p->n_probe < 0 || p->n_probe > N) return fail(SPARSEPR_ERR_INVALID_ARG, "n_probe must be in [0, N]");
  if (p->route_budget != SPARSEPR_BUDGET_UNIFORM && p->route_budget != SPARSEPR_BUDGET_GLOBAL)
    return fail(SPARSEPR_ERR_INVALID_ARG, "unknown route_budget %d", p->route_budget);
  if (p->route_budget == SPARSEPR_BUDGET_GLOBAL && spr::ceil_div(N, p->block) > 8192)
    return fail(SPARSEPR_ERR_UNSUPPORTED, "more than 8192 groups per head under the global budget is not built");
  const int G = spr::ceil_div(N, p->block);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const long long probe_pairs = static_cast<long long>(p->n_probe) * N;
  if (p->route_budget == SPARSEPR_BUDGET_GLOBAL) {
    // floor(rho N^2 - P N) in IEEE double, in this order
    if (!std::isfinite(p->density)) return fail(SPARSEPR_ERR_INVALID_ARG, "density must be finite");
    double budget = std::floor(p->density * static_cast<double>(N) * static_cast<double>(N) -
                               static_cast<double>(probe_pairs));
    // a head has at most N^2 <= 2^60 pairs: clamping the budget there changes no decision
    budget = std::min(std::max(budget, -0x1p61), 0x1p61);
    if (k_out) *k_out = G;
    SPR_CUDA(spr::launch_route_global(block_scores, Bt * H, G, G, static_cast<long long>(budget), route, key_gsize,
                                      qblock_size, reinterpret_cast<long long*>(executed_pairs), probe_pairs,
                                      &header(ws)->status, st),
             "route");
    return SPARSEPR_OK;
  }
  const int k = sparsepr_route_k(N, p->block, p->density, p->n_probe);
  if (k_out) *k_out = k;
  SPR_CUDA(spr::launch_route(block_scores, Bt * H, G, G, k, route, key_gsize, qblock_size,
                             reinterpret_cast<long long*>(executed_pairs), probe_pairs, &header(ws)->status, st),
           "route");
  return SPARSEPR_OK;
}

// Status word for attention calls made without a workspace (the dense comparator).
__device__ int g_attention_status_sink;

static int attention_common(const void* Q, const void* K, const void* V, int dtype, int32_t Bt, int32_t H,
                            int32_t N, int32_t d, int32_t block, const int32_t* key_perm, const int32_t* key_gsize,
                            const int32_t* query_perm, const int32_t* qblock_size, const int32_t* route, int32_t k,
                            float scale, float* out, bool dense, void* ws, sparsepr_stream_t stream) {
  int rc;
  if ((rc = check_shape(Bt, H, N, d)) || (rc = check_dtype(dtype)) || (rc = check_block(block))) return rc;
  if (!Q || !K || !V || !out) return fail(SPARSEPR_ERR_INVALID_ARG, "null pointer argument");
  if ((rc = check_aligned({Q, K, V}))) return rc;
  const int G = spr::ceil_div(N, block);
  if (!dense) {
    if (!key_perm || !key_gsize || !query_perm || !qblock_size || !route)
      return fail(SPARSEPR_ERR_INVALID_ARG, "null partition or route");
    if (k < 1 || k > G) return fail(SPARSEPR_ERR_INVALID_ARG, "k=%d outside [1, %d]", k, G);
  }
  spr::AttnArgs a{};
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.f32 = dtype == SPARSEPR_F32;
  a.heads = Bt * H;
  a.N = N;
  a.d = d;
  a.block = block;
  a.G = G;
  a.k = dense ? G : k;
  a.key_perm = key_perm;
  a.key_gsize = key_gsize;
  a.query_perm = query_perm;
  a.qblock_size = qblock_size;
  a.route = route;
  a.scale_log2 = resolve_scale(scale, d) * kLog2e;
  a.out = out;
  if (!dense && !a.f32 && d == 128 && block == 128) {
    if (ws == nullptr) return fail(SPARSEPR_ERR_INVALID_ARG, "sparse attention needs the workspace");
    const Layout L = make_layout(Bt * H, N, d, block, 1, 0);
    a.k_grouped = at<char>(ws, L.kv_grouped);
    a.v_grouped = at<char>(ws, L.kv_grouped) + static_cast<size_t>(Bt) * H * G * block * d * 2;
    a.kv_tag = header(ws)->kv_tag;
  }
  if (ws != nullptr) {
    a.status = &header(ws)->status;
  } else {
    SPR_CUDA(cudaGetSymbolAddress(reinterpret_cast<void**>(&a.status), g_attention_status_sink), "status sink");
  }
  SPR_CUDA(spr::launch_attention(a, dense, reinterpret_cast<cudaStream_t>(stream)), dense ? "dense attention" : "sparse attention");
  return SPARSEPR_OK;
}

int sparsepr_sparse_attn(const void* Q, const void* K, const void* V, int dtype, int32_t Bt, int32_t H, int32_t N,
                         int32_t d, int32_t block, const int32_t* key_perm, const int32_t* key_gsize,
                         const int32_t* query_perm, const int32_t* qblock_size, const int32_t* route, int32_t k,
                         float scale, float* S_out, void* ws, sparsepr_stream_t stream) {
  return attention_common(Q, K, V, dtype, Bt, H, N, d, block, key_perm, key_gsize, query_perm, qblock_size, route, k,
                          scale, S_out, false, ws, stream);
}

int sparsepr_sparse_attn_apply(const void* Q, const void* K, const void* V, int dtype, int32_t Bt, int32_t H,
                               int32_t N, int32_t d, int32_t block, const int32_t* key_perm, const int32_t* key_gsize,
                               const int32_t* query_perm, const int32_t* qblock_size, const int32_t* route, int32_t k,
                               float scale, const float* M, const float* beta, const int32_t* probe_idx, int32_t P,
                               const float* probe_out, void* O, void* ws, sparsepr_stream_t stream) {
  int rc;
  if ((rc = check_shape(Bt, H, N, d)) || (rc = check_dtype(dtype)) || (rc = check_block(block))) return rc;
  if (dtype != SPARSEPR_BF16 || d != 128 || block != 128)
    return fail(SPARSEPR_ERR_UNSUPPORTED, "the fused correction is built for bf16, d = 128, block = 128");
  if (!Q || !K || !V || !key_perm || !key_gsize || !query_perm || !qblock_size || !route || !M || !beta || !O || !ws)
    return fail(SPARSEPR_ERR_INVALID_ARG, "null pointer argument");
  if ((rc = check_aligned({Q, K, V}))) return rc;
  if (P < 0 || P > N || (P > 0 && (!probe_idx || !probe_out))) return fail(SPARSEPR_ERR_INVALID_ARG, "bad probe rows");
  const int G = spr::ceil_div(N, block);
  if (k < 1 || k > G) return fail(SPARSEPR_ERR_INVALID_ARG, "k=%d outside [1, %d]", k, G);
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const int heads = Bt * H;
  const Layout L = make_layout(heads, N, d, block, 1, 0);
  __nv_bfloat16* mh = at<__nv_bfloat16>(ws, L.mhilo);
  SPR_CUDA(spr::launch_split_bf16(M, mh, mh + static_cast<size_t>(heads) * d * d, static_cast<size_t>(heads) * d * d, st),
           "split M");
  spr::AttnArgs a{};
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.f32 = false;
  a.heads = heads;
  a.N = N;
  a.d = d;
  a.block = block;
  a.G = G;
  a.k = k;
  a.key_perm = key_perm;
  a.key_gsize = key_gsize;
  a.query_perm = query_perm;
  a.qblock_size = qblock_size;
  a.route = route;
  a.scale_log2 = resolve_scale(scale, d) * kLog2e;
  a.out = nullptr;
  a.status = &header(ws)->status;
  a.k_grouped = at<char>(ws, L.kv_grouped);
  a.v_grouped = at<char>(ws, L.kv_grouped) + static_cast<size_t>(heads) * G * block * d * 2;
  a.kv_tag = header(ws)->kv_tag;
  a.m_hilo = mh;
  a.beta = beta;
  a.out_bf16 = O;
  SPR_CUDA(spr::launch_attention(a, false, st), "sparse attention with correction");
  SPR_CUDA(spr::launch_probe_overwrite_bf16(probe_idx, probe_out, heads, N, P, static_cast<__nv_bfloat16*>(O), st),
           "probe rows");
  return SPARSEPR_OK;
}

int sparsepr_dense_attn(const void* Q, const void* K, const void* V, int dtype, int32_t Bt, int32_t H, int32_t N,
                        int32_t d, int32_t block, float scale, float* O_out, void* ws, sparsepr_stream_t stream) {
  return attention_common(Q, K, V, dtype, Bt, H, N, d, block, nullptr, nullptr, nullptr, nullptr, nullptr, 0, scale,
                          O_out, true, ws, stream);
}

int sparsepr_probe_dense(const void* Q, const void* K, const void* V, int dtype, int32_t Bt, int32_t H, int32_t N,
                         int32_t d, int32_t block, const int32_t* probe_idx, int32_t P, const int32_t* key_perm,
                         const int32_t* key_gsize, const int32_t* query_perm, const int32_t* route, int32_t k,
                         float scale, float* probe_out, float* probe_sparse, void* ws, sparsepr_stream_t stream) {
  int rc;
  if ((rc = check_shape(Bt, H, N, d)) || (rc = check_dtype(dtype)) || (rc = check_block(block))) return rc;
  if (P < 1 || P > N) return fail(SPARSEPR_ERR_INVALID_ARG, "P must be in [1, N]");
  if (!Q || !K || !V || !probe_idx || !key_perm || !key_gsize || !query_perm || !route || !probe_out ||
      !probe_sparse || !ws)
    return fail(SPARSEPR_ERR_INVALID_ARG, "null pointer argument");
  if ((rc = check_aligned({Q, K, V}))) return rc;
  const int G = spr::ceil_div(N, block);
  if (k < 1 || k > G) return fail(SPARSEPR_ERR_INVALID_ARG, "k=%d outside [1, %d]", k, G);
  const Layout L = make_layout(Bt * H, N, d, block, 1, P);
  spr::ProbeArgs a{};
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.f32 = dtype == SPARSEPR_F32;
  a.heads = Bt * H;
  a.N = N;
  a.d = d;
  a.block = block;
  a.G = G;
  a.k = k;
  a.P = P;
  a.probe_idx = probe_idx;
  a.key_perm = key_perm;
  a.key_gsize = key_gsize;
  a.query_perm = query_perm;
  a.route = route;
  a.scale_log2 = resolve_scale(scale, d) * kLog2e;
  a.probe_out = probe_out;
  a.probe_sparse = probe_sparse;
  a.qblk = at<int>(ws, L.qblk);
  a.partial = at<float>(ws, L.partial);
  a.k_grouped = at<char>(ws, L.kv_grouped);
  a.v_grouped = at<char>(ws, L.kv_grouped) + static_cast<size_t>(Bt) * H * G * block * d * 2;
  a.kv_tag = header(ws)->kv_tag;
  a.status = &header(ws)->status;
  SPR_CUDA(spr::launch_probe(a, reinterpret_cast<cudaStream_t>(stream)), "probe rows");
  return SPARSEPR_OK;
}

int sparsepr_fit_residual(const float* probe_sparse, const float* probe_out, const float* weights, int32_t Bt,
                          int32_t H, int32_t d, int32_t P, double ridge_lambda, int32_t rank, int32_t weight_mode,
                          float* M, float* beta, void* ws, sparsepr_stream_t stream) {
  int rc;
  if ((rc = check_shape(Bt, H, 1, d))) return rc;
  if (P < 1) return fail(SPARSEPR_ERR_INVALID_ARG, "P must be >= 1");
  if (rank < 1) return fail(SPARSEPR_ERR_INVALID_ARG, "rank must be >= 1");
  if (!(ridge_lambda >= 0.0)) return fail(SPARSEPR_ERR_INVALID_ARG, "ridge_lambda must be >= 0");
  if ((rc = check_weight_mode(weight_mode))) return rc;
  if (!probe_sparse || !probe_out || !M || !beta || !ws) return fail(SPARSEPR_ERR_INVALID_ARG, "null pointer argument");
  if (spr::fit_smem_bytes(d, P) > 220 * 1024) return fail(SPARSEPR_ERR_UNSUPPORTED, "P=%d too large for the fit", P);
  // The fit's scratch is the workspace's first region after the header (sized for the
  // largest P the fit takes, so its offset needs neither N nor the block); the key-group
  // K/V copy behind it stays intact for the attention call that follows.
  const size_t off = align_up(sizeof(spr::WorkspaceHeader));
  double* scratch = at<double>(ws, off);
  SPR_CUDA(spr::launch_fit(probe_sparse, probe_out, weights, Bt * H, d, P, ridge_lambda, rank, weight_mode, scratch, M,
                           beta, &header(ws)->status, reinterpret_cast<cudaStream_t>(stream)),
           "fit");
  return SPARSEPR_OK;
}

int sparsepr_apply_residual(const float* S_out, const float* M, const float* beta, const int32_t* probe_idx,
                            const float* probe_out, int32_t Bt, int32_t H, int32_t N, int32_t d, int32_t P, void* O,
                            int out_dtype, sparsepr_stream_t stream) {
  int rc;
  if ((rc = check_shape(Bt, H, N, d)) || (rc = check_dtype(out_dtype))) return rc;
  if (P < 0 || P > N) return fail(SPARSEPR_ERR_INVALID_ARG, "P must be in [0, N]");
  if (!S_out || !M || !beta || !O || (P > 0 && (!probe_idx || !probe_out)))
    return fail(SPARSEPR_ERR_INVALID_ARG, "null pointer argument");
  if (O == static_cast<const void*>(S_out) && out_dtype != SPARSEPR_F32)
    return fail(SPARSEPR_ERR_INVALID_ARG, "in-place apply needs out_dtype F32");
  SPR_CUDA(spr::launch_apply(S_out, M, beta, probe_idx, probe_out, Bt * H, N, d, P, O, out_dtype == SPARSEPR_F32,
                             reinterpret_cast<cudaStream_t>(stream)),
           "apply");
  return SPARSEPR_OK;
}

int sparsepr_probe_rows(int32_t N, int32_t P, int32_t Bt, int32_t H, int32_t* probe_idx,
                        sparsepr_stream_t stream) {
  if (N < 1 || P < 1 || P > N || Bt < 1 || H < 1 || !probe_idx)
    return fail(SPARSEPR_ERR_INVALID_ARG, "bad probe-row arguments");
  SPR_CUDA(spr::launch_probe_rows(N, P, Bt * H, probe_idx, reinterpret_cast<cudaStream_t>(stream)), "probe rows");
  return SPARSEPR_OK;
}

uint64_t sparsepr_launch_count(void) { return spr::g_launches.load(std::memory_order_relaxed); }

int sparsepr_kernel_timing(int enable) {
  spr::attn_timing_enable(enable != 0);
  return SPARSEPR_OK;
}

int sparsepr_kernel_timing_read(double* ms_total, int64_t* launches) {
  long long n = 0;
  double ms = 0.0;
  SPR_CUDA(spr::attn_timing_read(&ms, &n), "kernel timing read");
  if (ms_total) *ms_total = ms;
  if (launches) *launches = n;
  return SPARSEPR_OK;
}

int sparsepr_row_errors(const void* O, int o_dtype, const float* O_ref, const int32_t* probe_idx, int32_t Bt,
                        int32_t H, int32_t N, int32_t d, int32_t P, float* err, sparsepr_stream_t stream) {
  int rc;
  if ((rc = check_shape(Bt, H, N, d)) || (rc = check_dtype(o_dtype))) return rc;
  if (!O || !O_ref || !err || (P > 0 && !probe_idx)) return fail(SPARSEPR_ERR_INVALID_ARG, "null pointer argument");
  SPR_CUDA(spr::launch_row_errors(O, o_dtype == SPARSEPR_F32, O_ref, Bt * H, N, d, probe_idx, P, err,
                                  reinterpret_cast<cudaStream_t>(stream)),
           "row errors");
  return SPARSEPR_OK;
}

size_t sparsepr_test_fill_workspace_size(int32_t H, int32_t n, int32_t G) {
  if (H < 1 || n < 1 || G < 1) return 0;
  const size_t h = H, nn = n, g = G;
  return align_up(sizeof(spr::WorkspaceHeader)) + align_up(4 * h * g * sizeof(int)) +
         align_up(h * ((g + 31) / 32) * sizeof(unsigned int)) +
         align_up(h * nn * sizeof(unsigned long long)) + 3 * align_up(h * nn * sizeof(int)) + align_up(4 * sizeof(int)) +
         align_up(h * nn * sizeof(float));
}

int sparsepr_test_fill(const float* D, int32_t H, int32_t n, int32_t G, int32_t cap, int32_t* labels, void* ws,
                       sparsepr_stream_t stream) {
  if (!D || !labels || !ws || H < 1 || n < 1 || G < 1 || cap < 1)
    return fail(SPARSEPR_ERR_INVALID_ARG, "bad fill arguments");
  if (static_cast<long long>(G) * cap < n) return fail(SPARSEPR_ERR_INVALID_ARG, "G * cap < n");
  if (G > 1024) return fail(SPARSEPR_ERR_UNSUPPORTED, "more than 1024 groups is not built");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t h = H, nn = n, g = G;
  size_t off = align_up(sizeof(spr::WorkspaceHeader));
  auto take = [&](size_t bytes) {
    const size_t a = off;
    off += align_up(bytes);
    return a;
  };
  spr::FillArgs fa{};
  fa.D = D;
  fa.ldd = G;
  fa.prop_g0 = nullptr;
  fa.prop_v0 = nullptr;
  fa.heads = H;
  fa.n = n;
  fa.G = G;
  fa.cap = cap;
  fa.labels = labels;
  const size_t grp = take(4 * h * g * sizeof(int));
  fa.room = at<int>(ws, grp);
  fa.cnt = fa.room + h * g;
  fa.offs = fa.cnt + h * g;
  fa.cursor = fa.offs + h * g;
  fa.closed = at<unsigned int>(ws, take(h * ((g + 31) / 32) * sizeof(unsigned int)));
  fa.bucket = at<unsigned long long>(ws, take(h * nn * sizeof(unsigned long long)));
  fa.list0 = at<int>(ws, take(h * nn * sizeof(int)));
  fa.list1 = at<int>(ws, take(h * nn * sizeof(int)));
  fa.prop_g = at<int>(ws, take(h * nn * sizeof(int)));
  fa.list_len = at<int>(ws, take(4 * sizeof(int)));
  fa.prop_v = at<float>(ws, take(h * nn * sizeof(float)));
  fa.hdr = header(ws);
  SPR_CUDA(cudaMemsetAsync(ws, 0, sizeof(spr::WorkspaceHeader), st), "fill: reset status");
  SPR_CUDA(spr::launch_fill(fa, st), "fill");
  return SPARSEPR_OK;
}

int sparsepr_test_topk(const float* Sc, int32_t H, int32_t Gq, int32_t G, int32_t k, int32_t* route, void* ws,
                       sparsepr_stream_t stream) {
  if (!Sc || !route || !ws || H < 1 || Gq < 1 || G < 1 || k < 1 || k > G)
    return fail(SPARSEPR_ERR_INVALID_ARG, "bad top-k arguments");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  SPR_CUDA(cudaMemsetAsync(ws, 0, sizeof(spr::WorkspaceHeader), st), "topk: reset status");
  SPR_CUDA(spr::launch_route(Sc, H, Gq, G, k, route, nullptr, nullptr, nullptr, 0, &header(ws)->status, st), "topk");
  return SPARSEPR_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------------------
// Allocation-free variant of the residual fit.
//
// Some callers cannot call cudaMalloc: an inference-engine plugin must run inside the
// memory plan its host engine fixed before execution, and a latency-critical serving loop
// cannot take cudaMalloc's implicit device synchronisation and unbounded latency.  This
// entry point takes its scratch from a fixed array compiled into the library instead of a
// caller workspace.  The array is file-scope and static: every GPU that loads the library
// holds it until the process exits.  Its host-side name is only a stand-in for the device
// array, so the device address is looked up once per device (with that device current)
// and that address is what the kernel receives.
namespace {

constexpr size_t kNoAllocScratchBytes = 32ull << 20;  // 32 MiB
constexpr size_t kNoAllocStatusBytes = 256;            // status word, cleared every call
constexpr int kNoAllocMaxDevices = 64;

__device__ __align__(256) unsigned char g_fit_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_noalloc_mutex;
void* g_noalloc_base[kNoAllocMaxDevices] = {};
void* g_noalloc_ctx[kNoAllocMaxDevices] = {};  // context the cached address belongs to

// The current context of the calling thread, through the driver entry point (the
// runtime has no call for it); nullptr when the entry point is unavailable.
void* current_context() {
  using GetCurrent = int (*)(void**);
  static GetCurrent fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<GetCurrent>(p);
  }();
  void* ctx = nullptr;
  if (fn == nullptr || fn(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of the static scratch array on the current device.  Looked up once per
// device, and again when the device's context has changed since (a cudaDeviceReset
// unloads the module, so the old address would point outside any live allocation).
int noalloc_scratch(void** base) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "fit_noalloc: current device");
  if (dev < 0 || dev >= kNoAllocMaxDevices) return fail(SPARSEPR_ERR_UNSUPPORTED, "device index %d too large", dev);
  void* ctx = current_context();  // nullptr before the runtime made a context current: look up again
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  if (g_noalloc_base[dev] == nullptr || ctx == nullptr || ctx != g_noalloc_ctx[dev]) {
    void* ptr = nullptr;
    e = cudaGetSymbolAddress(&ptr, g_fit_noalloc_scratch);
    if (e != cudaSuccess) return cuda_fail(e, "fit_noalloc: scratch address");
    g_noalloc_base[dev] = ptr;
    g_noalloc_ctx[dev] = ctx;
  }
  *base = g_noalloc_base[dev];
  return SPARSEPR_OK;
}

}  // namespace

extern "C" int sparsepr_fit_residual_noalloc(const float* probe_sparse, const float* probe_out, const float* weights,
                                             int32_t Bt, int32_t H, int32_t d, int32_t P, double ridge_lambda,
                                             int32_t rank, int32_t weight_mode, float* M, float* beta,
                                             int32_t* status, sparsepr_stream_t stream) {
  int rc;
  if ((rc = check_shape(Bt, H, 1, d))) return rc;
  if (P < 1) return fail(SPARSEPR_ERR_INVALID_ARG, "P must be >= 1");
  if (rank < 1) return fail(SPARSEPR_ERR_INVALID_ARG, "rank must be >= 1");
  if (!(ridge_lambda >= 0.0)) return fail(SPARSEPR_ERR_INVALID_ARG, "ridge_lambda must be >= 0");
  if ((rc = check_weight_mode(weight_mode))) return rc;
  if (!probe_sparse || !probe_out || !M || !beta) return fail(SPARSEPR_ERR_INVALID_ARG, "null pointer argument");
  if (spr::fit_smem_bytes(d, P) > 220 * 1024) return fail(SPARSEPR_ERR_UNSUPPORTED, "P=%d too large for the fit", P);
  const size_t need = kNoAllocStatusBytes + sizeof(double) * static_cast<size_t>(Bt) * H * spr::fit_scratch_doubles(P, d);
  if (need > kNoAllocScratchBytes)
    return fail(SPARSEPR_ERR_UNSUPPORTED,
                "fit_noalloc: Bt*H=%d heads at d=%d, P=%d need %zu bytes of scratch; the fixed array holds %zu",
                Bt * H, d, P, need, kNoAllocScratchBytes);
  void* base = nullptr;
  if ((rc = noalloc_scratch(&base))) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  SPR_CUDA(cudaMemsetAsync(base, 0, kNoAllocStatusBytes, st), "fit_noalloc: clear status");
  double* scratch = reinterpret_cast<double*>(static_cast<char*>(base) + kNoAllocStatusBytes);
  SPR_CUDA(spr::launch_fit(probe_sparse, probe_out, weights, Bt * H, d, P, ridge_lambda, rank, weight_mode, scratch, M,
                           beta, static_cast<int*>(base), st),
           "fit_noalloc");
  if (status != nullptr)
    SPR_CUDA(cudaMemcpyAsync(status, base, sizeof(int32_t), cudaMemcpyDeviceToDevice, st), "fit_noalloc: status");
  return SPARSEPR_OK;
}
