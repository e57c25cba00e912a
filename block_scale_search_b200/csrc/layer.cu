// layer.cu -- a layer's projections in one call: the diagonal Hessian of every
// calibration input, the global scale of every weight and the windowed sweep
// of every weight, with the HBM-bound reductions streamed beside the
// FP32-bound sweeps.
//
// The results are those of the per-step calls (nvfp4_diag_hessian,
// nvfp4_global_scale, nvfp4_scale_sweep_quantize) on the same inputs, bit for
// bit: the side reductions (side_reduce.cuh) write the standalone kernels'
// partials in their order, and the standalone finalize kernels run on them.
//
// The weights are swept in the order with the lowest estimated time
// (plan_cost below: every permutation for up to four weights, otherwise each
// weight first with the others in the caller's order; ties keep the
// caller's order); every order writes the same bytes.  Schedule, on one stream, for
// the weights w_0 .. w_{n-1} in that order:
//   * a reduction's deadline is the first sweep that needs it: S of w_j is
//     needed by sweep j, h of an input by the first sweep of a weight using it
//     (inputs no weight uses: after the last sweep);
//   * reductions with deadline 0 (w_0's S and its input's h) run as the
//     standalone kernels first;
//   * every other reduction is spread over the sweeps before its deadline that
//     can carry side work, in contiguous task ranges, filling those sweeps in
//     proportion to their size (earliest deadlines first), and finalized right
//     after the last sweep carrying part of it;
//   * a reduction with no carrier before its deadline, or whose carrier could
//     not launch as one (stream capture: no counter slot), runs as the
//     standalone kernels instead (for such a carrier, right after its sweep).
#include <algorithm>
#include <vector>

#include "nvfp4_kernels.cuh"
#include "side_reduce.cuh"

namespace nvfp4 {

namespace {

size_t align256(size_t x) { return (x + 255) & ~size_t{255}; }

struct Reduction {
  int kind = 0;            // 0: h of input `idx`; 1: S of weight `idx`
  int idx = 0;
  int deadline = 0;        // first sweep that needs it (nw: none)
  LanePlan plan;           // the standalone kernel's lane grid
  int64_t side_R = 1;      // row lanes of the side task grid
  int64_t tasks = 0;       // side_R x V
  double bytes = 0.0;      // bytes read
  size_t ws_off = 0;       // standalone workspace (diag: partials R x in)
  int last_carrier = -1;   // last sweep carrying part of it
  bool standalone = false; // computed by the standalone kernels
};

struct Share {
  int red;                 // reduction index
  int64_t t0, t1;          // task range
};

struct Plan {
  std::vector<Reduction> red;
  std::vector<std::vector<Share>> shares;  // per sweep
  size_t amax_off = 0;     // nw words for carried absmax reductions
  size_t bytes = 0;
};

Plan make_plan(const LayerWeight* w, int nw, const LayerInput* x, int nx, int sms) {
  Plan P;
  size_t off = 0;
  // inputs' h
  for (int k = 0; k < nx; ++k) {
    Reduction r;
    r.kind = 0;
    r.idx = k;
    r.deadline = nw;
    for (int j = 0; j < nw; ++j)
      if (w[j].input == k) { r.deadline = j; break; }
    r.plan = diag_hessian_plan(x[k].tokens, x[k].in, sms);
    r.side_R = r.plan.R;  // the standalone grid, so the partials are the same
    r.tasks = x[k].tokens > 0 ? r.side_R * (x[k].in / 8) : 0;
    r.bytes = 2.0 * static_cast<double>(x[k].tokens) * static_cast<double>(x[k].in);
    r.ws_off = off;
    off = align256(off + diag_hessian_workspace_bytes(r.plan, x[k].in));
    P.red.push_back(r);
  }
  // weights' S
  for (int j = 0; j < nw; ++j) {
    Reduction r;
    r.kind = 1;
    r.idx = j;
    r.deadline = j;
    r.plan = global_scale_plan(w[j].out, w[j].in, sms);
    // a maximum does not depend on the grid: runs of at least 512 rows keep
    // each side task long next to its ring's fill and drain
    r.side_R = std::max<int64_t>(1, std::min<int64_t>(r.plan.R, w[j].out / 512));
    r.tasks = r.side_R * (w[j].in / 8);
    r.bytes = 2.0 * static_cast<double>(w[j].out) * static_cast<double>(w[j].in);
    r.ws_off = off;
    off = align256(off + std::max<size_t>(global_scale_workspace_bytes(r.plan), 4));
    P.red.push_back(r);
  }
  P.amax_off = off;
  off = align256(off + static_cast<size_t>(nw) * sizeof(uint32_t));
  P.bytes = off;

  // spread the reductions over the sweeps before their deadlines
  P.shares.assign(nw, {});
  std::vector<double> load(nw, 0.0), cap(nw, 0.0);
  std::vector<bool> carrier(nw, false);
  for (int j = 0; j < nw; ++j) {
    carrier[j] = sweep_can_carry(w[j].out, w[j].in, sms);
    cap[j] = static_cast<double>(w[j].out) * static_cast<double>(w[j].in);
  }
  std::vector<int> order(P.red.size());
  for (size_t i = 0; i < order.size(); ++i) order[i] = static_cast<int>(i);
  std::stable_sort(order.begin(), order.end(),
                   [&](int a, int b) { return P.red[a].deadline < P.red[b].deadline; });
  for (int ri : order) {
    Reduction& r = P.red[ri];
    std::vector<int> cs;
    for (int j = 0; j < r.deadline && j < nw; ++j)
      if (carrier[j] && P.shares[j].size() < static_cast<size_t>(kMaxSideJobs)) cs.push_back(j);
    if (r.deadline == 0 || r.tasks == 0 || cs.empty()) {
      r.standalone = true;
      continue;
    }
    // water-filling: the level L at which sum_j max(0, L cap_j - load_j) = bytes
    double lo = 0.0, hi = 1.0;
    auto fill = [&](double L) {
      double s = 0.0;
      for (int j : cs) s += std::max(0.0, L * cap[j] - load[j]);
      return s;
    };
    while (fill(hi) < r.bytes) hi *= 2.0;
    for (int it = 0; it < 100; ++it) {
      const double mid = 0.5 * (lo + hi);
      (fill(mid) < r.bytes ? lo : hi) = mid;
    }
    // contiguous task ranges in carrier order, sized by each carrier's amount
    int64_t t = 0;
    double acc = 0.0;
    for (size_t c = 0; c < cs.size(); ++c) {
      const int j = cs[c];
      const double amt = std::max(0.0, hi * cap[j] - load[j]);
      acc += amt;
      int64_t t_end = c + 1 == cs.size()
                          ? r.tasks
                          : static_cast<int64_t>(static_cast<double>(r.tasks) * std::min(1.0, acc / r.bytes));
      t_end = std::min(std::max(t_end, t), r.tasks);
      if (t_end > t) {
        P.shares[j].push_back(Share{ri, t, t_end});
        load[j] += r.bytes * static_cast<double>(t_end - t) / static_cast<double>(r.tasks);
        r.last_carrier = std::max(r.last_carrier, j);
      }
      t = t_end;
    }
    if (r.last_carrier < 0) r.standalone = true;
  }
  return P;
}

// A plan's time as HBM-byte equivalents: a reduction run on its own costs its
// bytes; a sweep of E weight elements and K candidates costs 1.3 E K (about
// 2.1e-13 s per element and candidate on B200, as long as 1.3 bytes take at
// the copy bandwidth), and carrying C bytes beside it max(that + 0.38 C, C)
// (a carrying sweep slows by about 38% of the carried reductions' own time).
double plan_cost(const Plan& P, const LayerWeight* w, int nw, int K) {
  constexpr double kSweepBytes = 1.3, kCarry = 0.38;
  double cost = 0.0;
  for (const Reduction& r : P.red)
    if (r.standalone) cost += r.bytes;
  for (int j = 0; j < nw; ++j) {
    double carried = 0.0;
    for (const Share& s : P.shares[j]) {
      const Reduction& r = P.red[s.red];
      if (!r.standalone && r.tasks > 0)
        carried += r.bytes * static_cast<double>(s.t1 - s.t0) / static_cast<double>(r.tasks);
    }
    const double sweep =
        static_cast<double>(w[j].out) * static_cast<double>(w[j].in) * K * kSweepBytes;
    cost += std::max(sweep + kCarry * carried, carried);
  }
  return cost;
}

}  // namespace

size_t layer_workspace_bytes(const LayerWeight* w, int nw, const LayerInput* x, int nx, int sms) {
  // the same for every order of the weights: each reduction's workspace is
  // sized and aligned on its own
  return make_plan(w, nw, x, nx, sms).bytes;
}

std::vector<int> layer_sweep_order(const LayerWeight* w, int nw, const LayerInput* x, int nx,
                                   int sms, int lo, int hi) {
  std::vector<int> perm(static_cast<size_t>(std::max(nw, 0)));
  for (int j = 0; j < nw; ++j) perm[j] = j;
  std::vector<int> best = perm;
  if (nw < 2) return best;
  const int K = hi - lo + 1;
  std::vector<LayerWeight> wp(static_cast<size_t>(nw));
  double best_cost = 0.0;
  bool first = true;
  // the caller's order is tried first; another must be cheaper by more than
  // rounding to replace it
  auto consider = [&](const std::vector<int>& order) {
    for (int j = 0; j < nw; ++j) wp[j] = w[order[j]];
    const double c = plan_cost(make_plan(wp.data(), nw, x, nx, sms), wp.data(), nw, K);
    if (first || c < best_cost * (1.0 - 1e-9)) {
      best_cost = c;
      best = order;
      first = false;
    }
  };
  if (nw <= kMaxOrderedWeights) {
    do consider(perm);
    while (std::next_permutation(perm.begin(), perm.end()));
  } else {
    // the first weight fixes the standalone prologue, where orders differ
    // most: each weight first, the others in the caller's order
    for (int f = 0; f < nw; ++f) {
      std::vector<int> order{f};
      for (int j = 0; j < nw; ++j)
        if (j != f) order.push_back(j);
      consider(order);
    }
  }
  return best;
}

cudaError_t quantize_layer(const LayerWeight* w_caller, int nw, const LayerInput* x, int nx,
                           float q_max, int lo, int hi, void* workspace, int sms,
                           const cudaEvent_t* events, cudaStream_t stream) {
  // the weights in the order they are swept; events stay indexed by the
  // caller's order
  const std::vector<int> perm = layer_sweep_order(w_caller, nw, x, nx, sms, lo, hi);
  std::vector<LayerWeight> wv(static_cast<size_t>(nw));
  for (int j = 0; j < nw; ++j) wv[j] = w_caller[perm[j]];
  const LayerWeight* w = wv.data();
  Plan P = make_plan(w, nw, x, nx, sms);
  char* ws = static_cast<char*>(workspace);
  uint32_t* words = reinterpret_cast<uint32_t*>(ws + P.amax_off);
  cudaError_t e = cudaSuccess;
  auto ok = [&](cudaError_t c) {
    if (e == cudaSuccess) e = c;
    return e == cudaSuccess;
  };
  // the standalone kernels of one reduction (partials and finalize)
  auto standalone = [&](int ri) {
    Reduction& r = P.red[ri];
    r.standalone = true;
    if (r.kind == 0) {
      const LayerInput& in = x[r.idx];
      return ok(launch_diag_hessian(in.X, in.tokens, in.in, in.ldx, in.h, 0,
                                    reinterpret_cast<float*>(ws + r.ws_off), r.plan, stream));
    }
    const LayerWeight& m = w[r.idx];
    return ok(launch_global_scale(m.W, m.out, m.ldw, q_max, m.S, m.amax, m.status,
                                  reinterpret_cast<uint32_t*>(ws + r.ws_off), r.plan, stream));
  };
  // carried absmax reductions fold into one zeroed word each
  if (!ok(cudaMemsetAsync(words, 0, static_cast<size_t>(nw) * sizeof(uint32_t), stream))) return e;
  for (size_t ri = 0; ri < P.red.size(); ++ri)
    if (P.red[ri].deadline == 0 && !standalone(static_cast<int>(ri))) return e;

  for (int j = 0; j < nw; ++j) {
    // reductions due now that nothing carried
    for (size_t ri = 0; ri < P.red.size(); ++ri) {
      const Reduction& r = P.red[ri];
      if (r.deadline == j && j > 0 && r.last_carrier < 0 && !standalone(static_cast<int>(ri)))
        return e;
    }
    const LayerWeight& m = w[j];
    const float* h = m.input >= 0 ? x[m.input].h : nullptr;
    bool carried = false;
    if (events != nullptr && !ok(cudaEventRecord(events[2 * perm[j]], stream))) return e;
    if (!P.shares[j].empty()) {
      SideWork sw{};
      sw.n = 0;
      sw.tasks = 0;
      for (const Share& s : P.shares[j]) {
        const Reduction& r = P.red[s.red];
        // an earlier carrier that could not carry ran this reduction whole
        if (r.standalone) continue;
        SideJob& jb = sw.job[sw.n++];
        if (r.kind == 0) {
          const LayerInput& in = x[r.idx];
          jb.A = in.X;
          jb.rows = in.tokens;
          jb.ld = in.ldx;
          jb.cols = in.in;
          jb.P = reinterpret_cast<float*>(ws + r.ws_off);
          jb.amax = nullptr;
        } else {
          const LayerWeight& o = w[r.idx];
          jb.A = o.W;
          jb.rows = o.out;
          jb.ld = o.ldw;
          jb.cols = o.in;
          jb.P = nullptr;
          jb.amax = words + r.idx;
        }
        jb.kind = r.kind;
        jb.R = r.side_R;
        jb.t0 = s.t0;
        jb.t1 = s.t1;
        sw.tasks += s.t1 - s.t0;
      }
      if (sw.n > 0 &&
          !ok(launch_scale_sweep_side(m.W, m.out, m.in, m.ldw, h, m.S, lo, hi, m.codes, m.scales,
                                      m.offs, sw, sms, &carried, stream)))
        return e;
    }
    if (!carried) {
      const LanePlan sp = sweep_plan(m.out, m.in, sms, h != nullptr, hi - lo + 1);
      if (!ok(launch_scale_sweep(m.W, m.out, m.in, m.ldw, h, m.S, lo, hi, m.codes, m.scales,
                                 m.offs, sp, stream)))
        return e;
    }
    if (events != nullptr && !ok(cudaEventRecord(events[2 * perm[j] + 1], stream))) return e;
    if (!carried) {
      // this sweep's shares: their reductions run whole, now
      for (const Share& s : P.shares[j])
        if (!P.red[s.red].standalone && !standalone(s.red)) return e;
    }
    // finalize what this sweep completed
    for (size_t ri = 0; ri < P.red.size(); ++ri) {
      const Reduction& r = P.red[ri];
      if (r.standalone || r.last_carrier != j) continue;
      if (r.kind == 0) {
        const LayerInput& in = x[r.idx];
        if (!ok(launch_diag_hessian_finalize(reinterpret_cast<const float*>(ws + r.ws_off),
                                             r.plan.R, in.in, in.h, 0, stream)))
          return e;
      } else {
        const LayerWeight& o = w[r.idx];
        if (!ok(launch_global_scale_finalize(words + r.idx, 1, q_max, o.S, o.amax, o.status,
                                             stream)))
          return e;
      }
    }
  }
  // inputs that no weight uses
  for (size_t ri = 0; ri < P.red.size(); ++ri) {
    const Reduction& r = P.red[ri];
    if (r.deadline == nw && r.last_carrier < 0 && !standalone(static_cast<int>(ri))) return e;
  }
  return e;
}

}  // namespace nvfp4
