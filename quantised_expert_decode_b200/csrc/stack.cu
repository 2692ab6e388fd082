// Layer stack: L x (route -> decode FFN) + residual RMSNorm, captured once into
// one CUDA graph whose arguments are fixed-address buffers in caller workspace.
#include <algorithm>
#include <new>
#include <vector>

#include "common.cuh"
#include "stack_fused.cuh"

namespace qmoe {
qmoe_status ffn_decode_launch(const qmoe_experts *ex, const float *x, int T, const int32_t *idx, const float *gate,
                              int k, float *y, void *ws, size_t ws_bytes, int32_t *status, cudaStream_t s,
                              bool cooperative);
}

struct qmoe_stack {
  int L, T, k, E, H, I, fmt;
  float eps;
  std::vector<const float *> Wr, bias;
  std::vector<qmoe_experts> layers;
  float *x_in, *x_out, *xa, *xb, *y;
  int32_t *idx;
  float *gate;
  int32_t *status;
  void *route_ws;
  size_t route_ws_bytes;
  void *ffn_ws;
  size_t ffn_ws_bytes;
  cudaGraph_t graph;
  cudaGraphExec_t exec;
  int kernels;
  int flags;
  int path;
  qmoe::FusedPlan fplan;
  qmoe::FusedBufs fbufs;
  std::vector<cudaEvent_t> events;  // 2L + 1 when timing
  long long *trace;                 // fused path with timing: [L][G][points] SM clock stamps
  int trace_ctas;
};

namespace {

size_t al(size_t b) { return (b + 255) & ~(size_t)255; }

struct Layout {
  size_t x, idx, gate, status, route, ffn, fused, trace, total;
  bool use_fused;
  qmoe::FusedPlan fplan;
};

// The stack's block format, or 0 when its layers mix formats.
int stack_fmt(const qmoe_stack_desc *d) {
  for (int l = 1; l < d->L; ++l)
    if (d->layers[l].fmt != d->layers[0].fmt) return 0;
  return d->layers[0].fmt;
}

Layout layout_of(const qmoe_stack_desc *d) {
  const qmoe_experts &e = d->layers[0];
  Layout l;
  const int fmt = stack_fmt(d);
  l.use_fused = d->T == 1 && !(d->flags & QMOE_STACK_LAYERWISE) &&
                qmoe::fused_stack_plan(fmt ? fmt : QMOE_Q4, e.E, e.H, e.I, d->k, &l.fplan);
  l.fused = l.use_fused ? al(qmoe::fused_stack_ws_bytes(d->L, e.E, e.H, e.I, d->k)) : 0;
  l.trace = (l.use_fused && (d->flags & QMOE_STACK_TIMING))
                ? al((size_t)d->L * qmoe::num_sms() * qmoe::fused_trace_points() * sizeof(long long))
                : 0;
  l.x = al((size_t)d->T * e.H * 4);
  l.idx = al((size_t)d->L * d->T * d->k * 4);
  l.gate = l.idx;
  l.status = 256;
  l.route = al(qmoe_route_workspace_bytes(d->T, e.E));
  l.ffn = al(qmoe_decode_workspace_bytes(d->T, d->k, e.H, e.I));
  l.total = 5 * l.x + l.idx + l.gate + l.status + l.route + l.ffn + l.fused + l.trace;
  return l;
}

qmoe_status check_desc(const qmoe_stack_desc *d) {
  if (!d || d->L < 1 || d->T < 1 || d->T > 8 || d->k < 1 || !d->Wr || !d->layers) return QMOE_ERR_INVALID_ARG;
  if (!(d->eps >= 0.0f)) return QMOE_ERR_INVALID_ARG;
  const qmoe_experts &e0 = d->layers[0];
  for (int l = 0; l < d->L; ++l) {
    const qmoe_experts &e = d->layers[l];
    if (e.E != e0.E || e.H != e0.H || e.I != e0.I) return QMOE_ERR_GEOMETRY;  // formats may differ
    if (e.fmt != QMOE_Q2 && e.fmt != QMOE_Q4) return QMOE_ERR_UNSUPPORTED;
    if (e.gate_up_bytes != qmoe_packed_bytes(e.fmt, QMOE_GATE_UP, e.E, e.H, e.I) ||
        e.down_bytes != qmoe_packed_bytes(e.fmt, QMOE_DOWN, e.E, e.H, e.I))
      return QMOE_ERR_GEOMETRY;
    if (!e.gate_up || !e.down || !d->Wr[l]) return QMOE_ERR_INVALID_ARG;
  }
  return QMOE_OK;
}

qmoe_status record(qmoe_stack *s, cudaStream_t cs, bool coop) {
  qmoe_status st;
  const float *x_prev = s->x_in;
  const bool timing = !s->events.empty();
  if (timing && cudaEventRecordWithFlags(s->events[0], cs, cudaEventRecordExternal) != cudaSuccess) return QMOE_ERR_CUDA;
  for (int l = 0; l < s->L; ++l) {
    int32_t *idx = s->idx + (size_t)l * s->T * s->k;
    float *gate = s->gate + (size_t)l * s->T * s->k;
    const float *bias = s->bias[l];
    const float *x_cur;
    if (l == 0) {
      st = qmoe_route(s->Wr[l], bias, s->x_in, QMOE_F32, s->T, s->H, s->E, s->k, idx, gate, s->route_ws,
                      s->route_ws_bytes, s->status, (qmoe_stream_t)cs);
      x_cur = s->x_in;
    } else {
      float *xo = (l & 1) ? s->xa : s->xb;
      st = qmoe_residual_route(x_prev, s->y, s->eps, xo, s->Wr[l], bias, s->T, s->H, s->E, s->k, idx, gate,
                               s->route_ws, s->route_ws_bytes, s->status, (qmoe_stream_t)cs);
      x_cur = xo;
    }
    if (st != QMOE_OK) return st;
    if (timing && cudaEventRecordWithFlags(s->events[2 * l + 1], cs, cudaEventRecordExternal) != cudaSuccess) return QMOE_ERR_CUDA;
    st = qmoe::ffn_decode_launch(&s->layers[l], x_cur, s->T, idx, gate, s->k, s->y, s->ffn_ws, s->ffn_ws_bytes,
                                 s->status, cs, coop);
    if (st != QMOE_OK) return st;
    if (timing && cudaEventRecordWithFlags(s->events[2 * l + 2], cs, cudaEventRecordExternal) != cudaSuccess) return QMOE_ERR_CUDA;
    x_prev = x_cur;
  }
  st = qmoe_rmsnorm_residual(x_prev, s->y, s->eps, s->x_out, s->T, s->H, (qmoe_stream_t)cs);
  s->kernels = 2 * s->L + 1;
  return st;
}

qmoe_status record_fused(qmoe_stack *s, cudaStream_t cs, bool coop) {
  const bool timing = !s->events.empty();
  if (timing && cudaEventRecordWithFlags(s->events[0], cs, cudaEventRecordExternal) != cudaSuccess) return QMOE_ERR_CUDA;
  qmoe_status st = qmoe::fused_launch(s->fbufs, s->fplan, s->fmt, s->L, s->E, s->H, s->I, s->k, s->eps, s->x_in,
                                      s->x_out, s->idx, s->gate, s->status, s->trace, cs, coop);
  if (st != QMOE_OK) return st;
  if (timing && cudaEventRecordWithFlags(s->events[1], cs, cudaEventRecordExternal) != cudaSuccess) return QMOE_ERR_CUDA;
  s->kernels = 1;
  return QMOE_OK;
}

qmoe_status capture(qmoe_stack *s, bool coop) {
  cudaStream_t cs;
  if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) return QMOE_ERR_CUDA;
  qmoe_status st = QMOE_OK;
  cudaGraph_t g = nullptr;
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaStreamDestroy(cs);
    return QMOE_ERR_CUDA;
  }
  qmoe_status rs = s->path == QMOE_PATH_FUSED ? record_fused(s, cs, coop) : record(s, cs, coop);
  cudaError_t e = cudaStreamEndCapture(cs, &g);
  if (rs != QMOE_OK) st = rs;
  else if (e != cudaSuccess) st = QMOE_ERR_CUDA;
  cudaGraphExec_t ex = nullptr;
  if (st == QMOE_OK && cudaGraphInstantiate(&ex, g, 0) != cudaSuccess) st = QMOE_ERR_CUDA;
  if (st == QMOE_OK) {
    s->graph = g;
    s->exec = ex;
  } else {
    if (g) cudaGraphDestroy(g);
    cudaGetLastError();
  }
  cudaStreamDestroy(cs);
  return st;
}

}  // namespace

extern "C" size_t qmoe_stack_workspace_bytes(const qmoe_stack_desc *d) {
  if (check_desc(d) != QMOE_OK) return 0;
  return layout_of(d).total;
}

extern "C" qmoe_status qmoe_stack_create(const qmoe_stack_desc *d, void *workspace, size_t workspace_bytes,
                                         qmoe_stream_t stream, qmoe_stack **out) {
  if (!out) return QMOE_ERR_INVALID_ARG;
  *out = nullptr;
  qmoe_status st = check_desc(d);
  if (st != QMOE_OK) return st;
  if (!workspace || !qmoe::aligned16(workspace)) return QMOE_ERR_INVALID_ARG;
  Layout lo = layout_of(d);
  if (workspace_bytes < lo.total) return QMOE_ERR_WORKSPACE;
  qmoe_stack *s = new (std::nothrow) qmoe_stack();
  if (!s) return QMOE_ERR_CUDA;
  const qmoe_experts &e0 = d->layers[0];
  s->L = d->L; s->T = d->T; s->k = d->k; s->E = e0.E; s->H = e0.H; s->I = e0.I; s->fmt = stack_fmt(d);
  s->eps = d->eps;
  s->Wr.assign(d->Wr, d->Wr + d->L);
  s->bias.assign(d->L, nullptr);
  if (d->bias)
    for (int l = 0; l < d->L; ++l) s->bias[l] = d->bias[l];
  s->layers.assign(d->layers, d->layers + d->L);
  s->flags = d->flags;
  if (d->flags & QMOE_STACK_TIMING) {
    s->events.assign(2 * d->L + 1, nullptr);
    for (auto &e : s->events)
      if (cudaEventCreate(&e) != cudaSuccess) {
        for (auto &e2 : s->events)
          if (e2) cudaEventDestroy(e2);
        delete s;
        return QMOE_ERR_CUDA;
      }
  }
  char *p = static_cast<char *>(workspace);
  s->x_in = reinterpret_cast<float *>(p); p += lo.x;
  s->x_out = reinterpret_cast<float *>(p); p += lo.x;
  s->xa = reinterpret_cast<float *>(p); p += lo.x;
  s->xb = reinterpret_cast<float *>(p); p += lo.x;
  s->y = reinterpret_cast<float *>(p); p += lo.x;
  s->idx = reinterpret_cast<int32_t *>(p); p += lo.idx;
  s->gate = reinterpret_cast<float *>(p); p += lo.gate;
  s->status = reinterpret_cast<int32_t *>(p); p += lo.status;
  s->route_ws = p; s->route_ws_bytes = lo.route; p += lo.route;
  s->ffn_ws = p; s->ffn_ws_bytes = lo.ffn; p += lo.ffn;
  s->path = lo.use_fused ? QMOE_PATH_FUSED : QMOE_PATH_LAYERWISE;
  s->fplan = lo.fplan;
  s->trace = nullptr;
  s->trace_ctas = 0;
  if (lo.use_fused) {
    s->fbufs = qmoe::fused_carve(p, d->L, s->E, s->H, s->I, s->k);
    p += lo.fused;
    if (lo.trace) {
      s->trace = reinterpret_cast<long long *>(p);
      s->trace_ctas = qmoe::num_sms();
    }
  }
  if (cudaMemsetAsync(workspace, 0, lo.total, (cudaStream_t)stream) != cudaSuccess ||
      cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) {
    delete s;
    return QMOE_ERR_CUDA;
  }
  if (s->path == QMOE_PATH_FUSED) {
    st = qmoe::fused_prepare(s->fbufs, s->L, s->E, s->H, d->Wr, d->layers, d->bias, (cudaStream_t)stream);
    if (st == QMOE_OK) {
      st = capture(s, true);                        // cooperative launch: all CTAs resident
      if (st == QMOE_ERR_CUDA) st = capture(s, false);
    }
  } else {
    st = capture(s, false);
  }
  if (st != QMOE_OK) {
    for (auto &e : s->events) cudaEventDestroy(e);
    delete s;
    return st;
  }
  *out = s;
  return QMOE_OK;
}

extern "C" qmoe_status qmoe_stack_destroy(qmoe_stack *s) {
  if (!s) return QMOE_ERR_INVALID_ARG;
  if (s->exec) cudaGraphExecDestroy(s->exec);
  if (s->graph) cudaGraphDestroy(s->graph);
  for (auto &e : s->events) cudaEventDestroy(e);
  delete s;
  return QMOE_OK;
}

extern "C" qmoe_status qmoe_stack_buffers(const qmoe_stack *s, float **x_in, float **x_out, int32_t **idx,
                                          float **gate, int32_t **dev_status) {
  if (!s) return QMOE_ERR_INVALID_ARG;
  if (x_in) *x_in = s->x_in;
  if (x_out) *x_out = s->x_out;
  if (idx) *idx = s->idx;
  if (gate) *gate = s->gate;
  if (dev_status) *dev_status = s->status;
  return QMOE_OK;
}

extern "C" int qmoe_stack_kernels_per_replay(const qmoe_stack *s) { return s ? s->kernels : 0; }

extern "C" uint32_t *qmoe_stack_barrier_word(const qmoe_stack *s) {
  return (s && s->path == QMOE_PATH_FUSED) ? s->fbufs.bar : nullptr;
}

extern "C" int qmoe_stack_path(const qmoe_stack *s) { return s ? s->path : -1; }

extern "C" qmoe_status qmoe_stack_decode(qmoe_stack *s, qmoe_stream_t stream) {
  if (!s || !s->exec) return QMOE_ERR_INVALID_ARG;
  cudaError_t e = cudaGraphLaunch(s->exec, (cudaStream_t)stream);
  qmoe::note_launch(s->kernels);
  return qmoe::cuda_status(e);
}

extern "C" qmoe_status qmoe_stack_decode_host(qmoe_stack *s, const float *x_host, float *x_out_host,
                                              qmoe_stream_t stream) {
  if (!s || !s->exec || !x_host || !x_out_host) return QMOE_ERR_INVALID_ARG;
  size_t bytes = (size_t)s->T * s->H * sizeof(float);
  cudaStream_t cs = (cudaStream_t)stream;
  if (cudaMemcpyAsync(s->x_in, x_host, bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess) return QMOE_ERR_CUDA;
  if (cudaGraphLaunch(s->exec, cs) != cudaSuccess) return QMOE_ERR_CUDA;
  qmoe::note_launch(s->kernels);
  if (cudaMemcpyAsync(x_out_host, s->x_out, bytes, cudaMemcpyDeviceToHost, cs) != cudaSuccess) return QMOE_ERR_CUDA;
  return QMOE_OK;
}

extern "C" qmoe_status qmoe_stack_layer_times(const qmoe_stack *s, float *route_ms, float *ffn_ms) {
  if (!s) return QMOE_ERR_INVALID_ARG;
  if (s->events.empty()) return QMOE_ERR_UNSUPPORTED;
  if (s->path == QMOE_PATH_FUSED) {
    // the kernel's event-timed duration, split over the layers in proportion
    // to each layer's median CTA clock span (start to start); route_ms is the
    // median span from a layer's start to its top-k
    float ms = 0.f;
    if (cudaEventSynchronize(s->events[1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms, s->events[0], s->events[1]) != cudaSuccess)
      return QMOE_ERR_CUDA;
    const int P = qmoe::fused_trace_points(), G = s->trace_ctas;
    std::vector<long long> tr((size_t)s->L * G * P);
    if (cudaMemcpy(tr.data(), s->trace, tr.size() * sizeof(long long), cudaMemcpyDeviceToHost) != cudaSuccess)
      return QMOE_ERR_CUDA;
    auto median = [](std::vector<double> v) {
      std::nth_element(v.begin(), v.begin() + v.size() / 2, v.end());
      return v[v.size() / 2];
    };
    std::vector<double> span(s->L), topk(s->L);
    double total = 0.0;
    for (int l = 0; l < s->L; ++l) {
      std::vector<double> a(G), b(G);
      for (int c = 0; c < G; ++c) {
        const long long *t = &tr[((size_t)l * G + c) * P];
        a[c] = (double)(t[6] - t[0]);   // layer start -> second grid barrier passed
        b[c] = (double)(t[1] - t[0]);   // layer start -> top-k done
      }
      span[l] = median(a);
      topk[l] = median(b);
      total += span[l];
    }
    for (int l = 0; l < s->L; ++l) {
      const double layer_ms = total > 0 ? ms * span[l] / total : ms / s->L;
      const double route = span[l] > 0 ? layer_ms * topk[l] / span[l] : 0.0;
      if (route_ms) route_ms[l] = (float)route;
      if (ffn_ms) ffn_ms[l] = (float)(layer_ms - route);
    }
    return QMOE_OK;
  }
  if (cudaEventSynchronize(s->events.back()) != cudaSuccess) return QMOE_ERR_CUDA;
  for (int l = 0; l < s->L; ++l) {
    float a = 0.f, b = 0.f;
    if (cudaEventElapsedTime(&a, s->events[2 * l], s->events[2 * l + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&b, s->events[2 * l + 1], s->events[2 * l + 2]) != cudaSuccess)
      return QMOE_ERR_CUDA;
    if (route_ms) route_ms[l] = a;
    if (ffn_ms) ffn_ms[l] = b;
  }
  return QMOE_OK;
}

extern "C" qmoe_status qmoe_stack_trace(const qmoe_stack *s, int64_t *cycles_host, size_t count, int *ctas,
                                        int *points) {
  if (!s || !cycles_host) return QMOE_ERR_INVALID_ARG;
  if (!s->trace) return QMOE_ERR_UNSUPPORTED;
  const int P = qmoe::fused_trace_points();
  const size_t n = (size_t)s->L * s->trace_ctas * P;
  if (count < n) return QMOE_ERR_WORKSPACE;
  if (cudaDeviceSynchronize() != cudaSuccess ||
      cudaMemcpy(cycles_host, s->trace, n * sizeof(long long), cudaMemcpyDeviceToHost) != cudaSuccess)
    return QMOE_ERR_CUDA;
  if (ctas) *ctas = s->trace_ctas;
  if (points) *points = P;
  return QMOE_OK;
}
