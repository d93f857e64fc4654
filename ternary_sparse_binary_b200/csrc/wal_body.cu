// Body-pass driver: every direct-packed body matrix of one decode step, run as
// one CUDA graph on one GPU.  The WAL-Ternary-8B runtime executes its decode
// step as a CUDA graph ("CUDA V18 Graph" in the speed table of the Kazakh
// README); here the graph holds the products of all body matrices in model
// order, grouped into dependency stages, as one persistent cooperative
// launch of the decode-GEMV kernel (groups of one stage back to back, a grid
// barrier between stages).
#include "wal_internal.h"
#include "wal_stream.h"

#include <cuda_runtime.h>

#include <atomic>

#include <algorithm>
#include <vector>

namespace wal {
int check_product_args(const wal_matrix* m, const void* X, int M, int ldx, const void* Y, int ldy);
StreamItem make_item(const wal_matrix* m, const uint16_t* x, float* y);
}  // namespace wal
using namespace wal;

struct wal_body_plan {
  int fmt = kFmtV1;
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

// Set by wal_debug_barrier_fault: plans built while it is nonzero get a grid
// barrier that no CTA reaches and a short wait limit.
std::atomic<int> g_barrier_fault{0};

bool same_matrix(const wal_matrix& a, const wal_matrix& b) {
  return a.N == b.N && a.K == b.K && a.k == b.k && a.r == b.r && a.codes == b.codes && a.sites == b.sites &&
         a.scales == b.scales && a.u_bits == b.u_bits && a.v_bits == b.v_bits && a.lr_scale == b.lr_scale;
}

bool plan_matches(const wal_body_plan* p, int fmt, const wal_matrix* mats, int n, const int32_t* stage_of,
                  const uint16_t* const* xs, float* const* ys, int M, void* ws, size_t ws_bytes) {
  if (!p || !p->exec || p->fmt != fmt || (int)p->mats.size() != n || p->M != M || p->ws != ws ||
      p->ws_bytes != ws_bytes)
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

// One group of the launch: products that share K, all in one dependency stage.
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

// Workspace of a body pass (offsets from the 256-byte aligned base):
// [0, 256) header: status word at 0, grid-barrier counter at 128;
// then the item table and the per-CTA schedules ([CTA][group] tile records)
// the persistent launch reads.  There are at most n_mats groups.
constexpr size_t kBarrierOffset = 128;
constexpr int kMaxCtas = 1024;
size_t items_offset() { return 256; }
size_t sched_offset(int n_mats, int M) { return align_up(256 + (size_t)n_mats * M * sizeof(StreamItem), 256); }
size_t body_ws_total(int n_mats, int M) {
  return 256 /*alignment slack*/ + sched_offset(n_mats, M) + (size_t)kMaxCtas * n_mats * sizeof(TileRec);
}

}  // namespace

namespace wal {

size_t body_workspace_total(int n_mats, int M) { return body_ws_total(n_mats, M); }

// A body pass over matrices of one format (kFmtPq2: codes point at PQ2_0
// block buffers, k = r = 0).  The caller has checked every argument.
int body_pass_impl(wal_body_plan** plan, int fmt, const wal_matrix* mats, int n_mats, const int32_t* stage_of,
                   const uint16_t* const* xs, float* const* ys, int M, void* ws, size_t ws_bytes,
                   cudaStream_t stream) {
  wal_body_plan* p = *plan;
  if (!plan_matches(p, fmt, mats, n_mats, stage_of, xs, ys, M, ws, ws_bytes)) {
    if (!p) {
      p = new wal_body_plan();
      cudaError_t e = cudaStreamCreateWithFlags(&p->capture_stream, cudaStreamNonBlocking);
      if (e != cudaSuccess) {
        delete p;
        return fail(WAL_ERR_CUDA, std::string("stream create: ") + cudaGetErrorString(e));
      }
      *plan = p;
    }
    // the previous graph may still be running on `stream` and reading the
    // launch tables in the workspace
    cudaError_t se = cudaStreamSynchronize((cudaStream_t)stream);
    if (se != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("stream synchronize: ") + cudaGetErrorString(se));
    release(p);
    p->fmt = fmt;
    p->mats.assign(mats, mats + n_mats);
    p->stages.assign(stage_of, stage_of + n_mats);
    p->xs.assign(xs, xs + n_mats);
    p->ys.assign(ys, ys + n_mats);
    p->M = M;
    p->ws = ws;
    p->ws_bytes = ws_bytes;

    // launch tables: groups and items, uploaded into the workspace
    const std::vector<LaunchGroup> lgs = group_launches(mats, n_mats, stage_of, M);
    std::vector<GroupDesc> groups(lgs.size());
    std::vector<StreamItem> items;
    items.reserve((size_t)n_mats * M);
    for (size_t gi = 0; gi < lgs.size(); ++gi) {
      const LaunchGroup& lg = lgs[gi];
      const int item0 = (int)items.size();
      for (int i = lg.first; i < lg.first + lg.count; ++i)
        for (int mi = 0; mi < M; ++mi)
          items.push_back(make_item(&mats[i], xs[i] + (size_t)mi * mats[i].K, ys[i] + (size_t)mi * mats[i].N));
      int st = plan_group(items.data() + item0, (int)items.size() - item0, mats[lg.first].K, &groups[gi]);
      if (st) return st;
      groups[gi].item0 = item0;
      // stages renumbered 0, 1, 2, ... (only changes matter to the launch)
      groups[gi].stage = gi == 0 ? 0 : groups[gi - 1].stage + (stage_of[lg.first] != stage_of[lgs[gi - 1].first]);
    }
    // A group right after a grid barrier may build its x image before the
    // barrier completes when no product of the stage before writes its x:
    // no x range of the group meets a y range of that stage.
    for (size_t gi = 1; gi < groups.size(); ++gi) {
      groups[gi].xfree = 0;
      if (groups[gi].stage == groups[gi - 1].stage) continue;
      bool overlap = false;
      for (size_t gk = 0; gk < gi && !overlap; ++gk) {
        if (groups[gk].stage != groups[gi - 1].stage) continue;
        for (int a = 0; a < groups[gk].n_items && !overlap; ++a) {
          const StreamItem& w = items[groups[gk].item0 + a];
          const uintptr_t y0 = (uintptr_t)w.y, y1 = y0 + (uintptr_t)w.N * 4u;
          for (int b = 0; b < groups[gi].n_items && !overlap; ++b) {
            const uintptr_t x0 = (uintptr_t)items[groups[gi].item0 + b].x;
            const uintptr_t x1 = x0 + (uintptr_t)groups[gi].K * 2u;
            overlap = x0 < y1 && y0 < x1;
          }
        }
      }
      groups[gi].xfree = overlap ? 0 : 1;
    }
    StreamLaunch L;
    int st = plan_launch(groups.data(), (int)groups.size(), true, fmt, &L);
    if (st) return st;
    if (L.grid > kMaxCtas) return fail(WAL_ERR_UNSUPPORTED, "more than 1024 SMs");
    const int ng = (int)groups.size();
    std::vector<TileRec> sched((size_t)L.grid * ng);
    for (int b = 0; b < L.grid; ++b) build_schedule(groups.data(), ng, items.data(), b, sched.data() + (size_t)b * ng);
    char* base = reinterpret_cast<char*>(align_up((uintptr_t)ws, 256));
    cudaError_t e = cudaMemcpy(base + items_offset(), items.data(), items.size() * sizeof(StreamItem),
                               cudaMemcpyHostToDevice);
    if (e == cudaSuccess)
      e = cudaMemcpy(base + sched_offset(n_mats, M), sched.data(), sched.size() * sizeof(TileRec),
                     cudaMemcpyHostToDevice);
    if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("launch-table upload: ") + cudaGetErrorString(e));
    StreamParams prm = {};
    prm.t_sched = reinterpret_cast<const TileRec*>(base + sched_offset(n_mats, M));
    prm.t_items = reinterpret_cast<const StreamItem*>(base + items_offset());
    prm.n_groups = ng;
    prm.barrier = reinterpret_cast<unsigned int*>(base + kBarrierOffset);
    prm.status = reinterpret_cast<int32_t*>(base);
    prm.fmt = fmt;
    if (g_barrier_fault.load()) {
      // fault injection: no CTA reaches a barrier target, and a wait gives up after 1 ms
      prm.barrier_bias = 1u << 30;
      prm.wait_ns = 1000000ull;
    }

    e = cudaStreamBeginCapture(p->capture_stream, cudaStreamCaptureModeThreadLocal);
    if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("begin capture: ") + cudaGetErrorString(e));
    // status word and barrier counter start at zero on every replay
    e = cudaMemsetAsync(base, 0, 256, p->capture_stream);
    if (e != cudaSuccess) st = fail(WAL_ERR_CUDA, std::string("header clear: ") + cudaGetErrorString(e));
    if (st == WAL_OK) st = launch_body(prm, L, p->capture_stream);
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
  cudaError_t e = cudaGraphLaunch(p->exec, stream);
  if (e != cudaSuccess) return fail(WAL_ERR_CUDA, std::string("graph launch: ") + cudaGetErrorString(e));
  return WAL_OK;
}

}  // namespace wal

extern "C" size_t wal_body_workspace_bytes(const wal_matrix* mats, int n_mats, int M) {
  if (!mats || n_mats <= 0 || M < 1) return 0;
  for (int i = 0; i < n_mats; ++i)
    if (!wal_workspace_bytes(&mats[i], M)) return 0;
  return body_ws_total(n_mats, M);
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
  return body_pass_impl(plan, kFmtV1, mats, n_mats, stage_of, xs, ys, M, ws, ws_bytes, (cudaStream_t)stream);
}

extern "C" int wal_debug_barrier_fault(int on) { return g_barrier_fault.exchange(on ? 1 : 0); }

extern "C" void wal_body_plan_destroy(wal_body_plan* plan) {
  if (!plan) return;
  release(plan);
  if (plan->capture_stream) cudaStreamDestroy(plan->capture_stream);
  delete plan;
}
