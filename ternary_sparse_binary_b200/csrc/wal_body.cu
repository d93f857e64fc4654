// Body-pass driver: every direct-packed body matrix of one decode step, run as
// one CUDA graph on one GPU.  The WAL-Ternary-8B runtime executes its decode
// step as a CUDA graph ("CUDA V18 Graph" in the speed table of the Kazakh
// README); here the graph holds the products of all body matrices in model
// order, grouped into dependency stages.
#include "wal_internal.h"
#include "wal_stream.h"

#include <cuda_runtime.h>

#include <algorithm>
#include <vector>

namespace wal {
int check_product_args(const wal_matrix* m, const void* X, int M, int ldx, const void* Y, int ldy);
StreamItem make_item(const wal_matrix* m, const uint16_t* x, float* y);
}  // namespace wal
using namespace wal;

struct wal_body_plan {
  std::vector<wal_matrix> mats;
  std::vector<int32_t> stages;
  std::vector<const uint16_t*> xs;
  std::vector<float*> ys;
  int M = 0;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  cudaStream_t capture_stream = nullptr;
  cudaGraph_t graph = nullptr;
  cudaGraphExec_t exec = nullptr;
};

namespace {

bool same_matrix(const wal_matrix& a, const wal_matrix& b) {
  return a.N == b.N && a.K == b.K && a.k == b.k && a.r == b.r && a.codes == b.codes && a.sites == b.sites &&
         a.scales == b.scales && a.u_bits == b.u_bits && a.v_bits == b.v_bits && a.lr_scale == b.lr_scale;
}

bool plan_matches(const wal_body_plan* p, const wal_matrix* mats, int n, const int32_t* stage_of,
                  const uint16_t* const* xs, float* const* ys, int M, void* ws, size_t ws_bytes) {
  if (!p || !p->exec || (int)p->mats.size() != n || p->M != M || p->ws != ws || p->ws_bytes != ws_bytes)
    return false;
  for (int i = 0; i < n; ++i)
    if (!same_matrix(p->mats[i], mats[i]) || p->stages[i] != stage_of[i] || p->xs[i] != xs[i] || p->ys[i] != ys[i])
      return false;
  return true;
}

void release(wal_body_plan* p) {
  if (p->exec) cudaGraphExecDestroy(p->exec);
  if (p->graph) cudaGraphDestroy(p->graph);
  p->exec = nullptr;
  p->graph = nullptr;
}

// One launch of the capture: products that share K, all in one dependency stage.
struct LaunchGroup {
  int first, count;  // matrices [first, first + count)
};

std::vector<LaunchGroup> group_launches(const wal_matrix* mats, int n, const int32_t* stage_of, int M) {
  std::vector<LaunchGroup> out;
  const int per_launch = std::max(1, kMaxItems / M);
  int i = 0;
  while (i < n) {
    int j = i + 1;
    while (j < n && stage_of[j] == stage_of[i] && mats[j].K == mats[i].K && j - i < per_launch) ++j;
    out.push_back({i, j - i});
    i = j;
  }
  return out;
}

int add_prefetch(PrefetchRange* pf, int n_pf, const void* p, size_t bytes) {
  if (!p || bytes == 0 || n_pf >= kMaxPrefetch) return n_pf;
  pf[n_pf].ptr = p;
  pf[n_pf].bytes = bytes & ~(size_t)15;
  return pf[n_pf].bytes ? n_pf + 1 : n_pf;
}

}  // namespace

extern "C" size_t wal_body_workspace_bytes(const wal_matrix* mats, int n_mats, int M) {
  if (!mats || n_mats <= 0 || M < 1) return 0;
  for (int i = 0; i < n_mats; ++i)
    if (!wal_workspace_bytes(&mats[i], M)) return 0;
  return 512;  // status header only: the batch-1 kernels keep every intermediate on chip
}

extern "C" int wal_body_pass(wal_body_plan** plan, const wal_matrix* mats, int n_mats, const int32_t* stage_of,
                             const uint16_t* const* xs, float* const* ys, int M, void* ws, size_t ws_bytes,
                             wal_stream_t stream) {
  if (!plan || !mats || !stage_of || !xs || !ys || n_mats <= 0)
    return fail(WAL_ERR_ARG, "plan, mats, stage_of, xs and ys are required and n_mats > 0");
  if (M < 1 || M > WAL_MAX_SMALL_M) return fail(WAL_ERR_SHAPE, "body pass supports 1 <= M <= 16");
  for (int i = 0; i < n_mats; ++i) {
    int st = check_product_args(&mats[i], xs[i], M, mats[i].K, ys[i], mats[i].N);
    if (st) return st;
    if (i && stage_of[i] < stage_of[i - 1]) return fail(WAL_ERR_ARG, "stage_of must be non-decreasing");
  }
  const size_t need = wal_body_workspace_bytes(mats, n_mats, M);
  if (!ws || ws_bytes < need) return fail(WAL_ERR_WORKSPACE, "body-pass workspace too small");

  wal_body_plan* p = *plan;
  if (!plan_matches(p, mats, n_mats, stage_of, xs, ys, M, ws, ws_bytes)) {
    if (!p) {
      p = new wal_body_plan();
      cudaError_t e = cudaStreamCreateWithFlags(&p->capture_stream, cudaStreamNonBlocking);
      if (e != cudaSuccess) {
        delete p;
        return fail(WAL_ERR_CUDA, std::string("stream create: ") + cudaGetErrorString(e));
      }
      *plan = p;
    }
    release(p);
    p->mats.assign(mats, mats + n_mats);
    p->stages.assign(stage_of, stage_of + n_mats);
    p->xs.assign(xs, xs + n_mats);
    p->ys.assign(ys, ys + n_mats);
    p->M = M;
    p->ws = ws;
    p->ws_bytes = ws_bytes;

    cudaError_t e = cudaStreamBeginCapture(p->capture_stream, cudaStreamCaptureModeThreadLocal);
    if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("begin capture: ") + cudaGetErrorString(e));
    int st = WAL_OK;
    const std::vector<LaunchGroup> groups = group_launches(mats, n_mats, stage_of, M);
    for (size_t gi = 0; gi < groups.size() && st == WAL_OK; ++gi) {
      const LaunchGroup& lg = groups[gi];
      StreamParams prm = {};
      prm.K = mats[lg.first].K;
      prm.status = reinterpret_cast<int32_t*>(align_up((uintptr_t)ws, 256));
      int n_items = 0;
      for (int i = lg.first; i < lg.first + lg.count; ++i)
        for (int mi = 0; mi < M; ++mi)
          prm.items[n_items++] = make_item(&mats[i], xs[i] + (size_t)mi * mats[i].K, ys[i] + (size_t)mi * mats[i].N);
      prm.n_items = n_items;
      // warm L2 with the weights of the next launch
      if (gi + 1 < groups.size()) {
        const LaunchGroup& nx = groups[gi + 1];
        int n_pf = 0;
        for (int i = nx.first; i < nx.first + nx.count; ++i) {
          size_t sz[6];
          sizes_of(mats[i].N, mats[i].K, mats[i].k, mats[i].r, sz);
          n_pf = add_prefetch(prm.pf, n_pf, mats[i].codes, sz[0]);
          n_pf = add_prefetch(prm.pf, n_pf, mats[i].sites, sz[1]);
          n_pf = add_prefetch(prm.pf, n_pf, mats[i].scales, sz[2]);
        }
        prm.n_pf = n_pf;
      }
      StreamLaunch L;
      st = plan_stream(prm.items, n_items, prm.K, &L);
      if (st == WAL_OK) st = launch_stream(prm, L, p->capture_stream, gi > 0);
    }
    cudaGraph_t g = nullptr;
    e = cudaStreamEndCapture(p->capture_stream, &g);
    if (st != WAL_OK) {
      if (g) cudaGraphDestroy(g);
      return st;
    }
    if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("end capture: ") + cudaGetErrorString(e));
    p->graph = g;
    e = cudaGraphInstantiate(&p->exec, g, 0);
    if (e != cudaSuccess) {
      release(p);
      return fail(WAL_ERR_CUDA, std::string("graph instantiate: ") + cudaGetErrorString(e));
    }
  }
  cudaError_t e = cudaGraphLaunch(p->exec, (cudaStream_t)stream);
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("graph launch: ") + cudaGetErrorString(e));
  return WAL_OK;
}

extern "C" void wal_body_plan_destroy(wal_body_plan* plan) {
  if (!plan) return;
  release(plan);
  if (plan->capture_stream) cudaStreamDestroy(plan->capture_stream);
  delete plan;
}
