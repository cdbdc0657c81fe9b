// C-ABI of the library (declared in include/fi.h): argument checks, device
// memory, and the host side of the relaxed schedule (which block runs at
// which step, and on which kernel).
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstring>
#include <new>
#include <string>
#include <vector>

#include "fi_internal.cuh"

using namespace fi;

namespace {

thread_local std::string g_last_error;

fi_status fail(fi_status s, const std::string& msg) {
  g_last_error = msg;
  return s;
}

fi_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FI_E_CUDA, std::string(what) + ": " + cudaGetErrorString(e));
}

#define FI_CUDA(call, what)                         \
  do {                                              \
    cudaError_t e_ = (call);                        \
    if (e_ != cudaSuccess) return cuda_fail(e_, what); \
  } while (0)

// fi_generate_host splits a generation into about kHostSegments segments of
// whole chunks (none shorter than kHostSegmentMin positions) so that copies
// overlap work.
constexpr int kHostSegments = 16;
constexpr int kHostSegmentMin = 256;

struct EventPair {
  cudaEvent_t a, b;
  int cls;
  int side_q;   // log2 of the block side for block launches, else -1
  int kernels;  // kernels the bracketed launch runs (a graph: its kernel nodes)
};

}  // namespace

void fi::set_last_error(const std::string& msg) { g_last_error = msg; }

struct fi_ctx {
  Dims g{};
  fi_config cfg{};
  cudaStream_t st = nullptr;
  int device = 0, num_sms = 0;
  size_t max_smem = 0;
  int pos = 0;
  int lazy_mode = 0;  // 1 after fi_generate_lazy until fi_reset
  int chunk = 0, fft_from = 0, q_lo = 0, q_hi = -1;
  int tc_q_hi = -1;                // block sides 2^6 .. 2^tc_q_hi run on the tensor cores
  TcPlan tc[32] = {};
  int chunk_G = 0;
  bool pdl_blocks = false;         // FFT blocks launched programmatically (the chunk grid fills the SMs)
  float* state = nullptr;
  float* taps = nullptr;
  float2* spectra = nullptr;
  float2* twiddle = nullptr;
  int* err = nullptr;      // device flag: a bounded wait in a kernel gave up
  int wait_limit = kDefaultWaitLimit;
  size_t spec_off[32] = {};
  float2* part_xs = nullptr;       // forward spectra of source sub-blocks (blocks wider than one transform)
  float2* pf_spec = nullptr;       // prompt prefill: padded filter spectra (allocated on first use)
  size_t pf_spec_n = 0;
  MlpBlock mlp;                    // channel-mixing block (hidden = 0: elementwise tanh)
  cudaGraphExec_t mlp_graph = nullptr;   // the block's layers at *mlp.pos, then the position advanced
  cudaStream_t cap_st = nullptr;         // capture stream for mlp_graph
  // staging for fi_generate_host
  void* d_x0 = nullptr;
  float* d_eps = nullptr;
  float* d_y = nullptr;
  size_t stage_n = 0;
  cudaStream_t up_st = nullptr, dn_st = nullptr;   // host copies of fi_generate_host, beside the work
  std::vector<cudaEvent_t> seg_ev;                 // per segment: uploaded, generated
  // profiling
  int prof = 0;
  std::vector<EventPair> ev_live, ev_free;
};

namespace {

bool pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

void free_mlp(fi_ctx* c) {
  if (c->mlp_graph) cudaGraphExecDestroy(c->mlp_graph);
  c->mlp_graph = nullptr;
  MlpBlock& m = c->mlp;
  cudaFree(m.w1);
  cudaFree(m.b1);
  cudaFree(m.w2);
  cudaFree(m.b2);
  cudaFree(m.z);
  cudaFree(m.y);
  cudaFree(m.pos);
  m = MlpBlock{};
}

void free_ctx(fi_ctx* c) {
  if (!c) return;
  free_mlp(c);
  if (c->cap_st) cudaStreamDestroy(c->cap_st);
  cudaFree(c->state);
  cudaFree(c->taps);
  cudaFree(c->spectra);
  cudaFree(c->part_xs);
  cudaFree(c->pf_spec);
  cudaFree(c->twiddle);
  cudaFree(c->err);
  cudaFree(c->d_x0);
  cudaFree(c->d_eps);
  cudaFree(c->d_y);
  for (cudaEvent_t e : c->seg_ev) cudaEventDestroy(e);
  if (c->up_st) cudaStreamDestroy(c->up_st);
  if (c->dn_st) cudaStreamDestroy(c->dn_st);
  for (auto& e : c->ev_live) { cudaEventDestroy(e.a); cudaEventDestroy(e.b); }
  for (auto& e : c->ev_free) { cudaEventDestroy(e.a); cudaEventDestroy(e.b); }
  delete c;
}

fi_status dev_alloc(void** p, size_t bytes, const char* what) {
  cudaError_t e = cudaMalloc(p, bytes);
  if (e != cudaSuccess) {
    cudaGetLastError();
    *p = nullptr;
    return fail(FI_E_OOM, std::string("cudaMalloc failed for ") + what + " (" + std::to_string(bytes) + " bytes): " +
                              cudaGetErrorString(e));
  }
  return FI_OK;
}

// Kernel launch wrapped in profiling events when enabled.
template <class F>
fi_status timed(fi_ctx* c, int cls, F&& launch, const char* what, int side_q = -1, int kernels = 1) {
  EventPair ep{};
  if (c->prof) {
    if (!c->ev_free.empty()) {
      ep = c->ev_free.back();
      c->ev_free.pop_back();
    } else {
      FI_CUDA(cudaEventCreate(&ep.a), "cudaEventCreate");
      FI_CUDA(cudaEventCreate(&ep.b), "cudaEventCreate");
    }
    ep.cls = cls;
    ep.side_q = side_q;
    ep.kernels = kernels;
    FI_CUDA(cudaEventRecord(ep.a, c->st), "cudaEventRecord");
  }
  cudaError_t e = launch();
  if (e != cudaSuccess) return cuda_fail(e, what);
  if (c->prof) {
    FI_CUDA(cudaEventRecord(ep.b, c->st), "cudaEventRecord");
    c->ev_live.push_back(ep);
  }
  return FI_OK;
}

// The block of step i (side U = lowbit(i)), read from and written to HBM.
// Targets below t_min are left alone (t_min <= i: the whole block); such
// partial blocks never go to the tensor cores.
fi_status run_block(fi_ctx* c, int i, int t_min = 0) {
  const int U = i & -i;
  const int q = ilog2((uint32_t)U);
  if (q > kMaxFftLog2 && c->q_lo <= kMaxFftLog2) {
    return timed(c, KC_FFT,
                 [&] {
                   return launch_part_block(c->g, c->state, c->part_xs, c->spectra + c->spec_off[q], c->twiddle, i,
                                            t_min, c->st);
                 },
                 "partitioned FFT block launch", q);
  }
  if (q >= kMinFftLog2 && q <= c->tc_q_hi && t_min <= i) {
    return timed(c, KC_TC,
                 [&] { return launch_tile_tc(c->g, c->state, c->taps, c->tc[q], i, c->err, c->wait_limit, c->st); },
                 "tensor-core block launch", q);
  }
  if (q >= c->q_lo && q <= c->q_hi) {
    return timed(c, KC_FFT,
                 [&] {
                   return launch_tile_fft(c->g, c->state, c->spectra + c->spec_off[q], c->twiddle, i, t_min, c->st,
                                          c->pdl_blocks);
                 },
                 "FFT block launch", q);
  }
  return timed(c, KC_DIRECT, [&] { return launch_tile_direct(c->g, c->state, c->taps, i, t_min, c->st); },
               "direct block launch", q);
}

// Synchronise the context's stream and report a device-side wait that gave up.
fi_status sync_and_check(fi_ctx* c) {
  FI_CUDA(cudaStreamSynchronize(c->st), "synchronize");
  int flag = 0;
  FI_CUDA(cudaMemcpy(&flag, c->err, sizeof(int), cudaMemcpyDeviceToHost), "read error flag");
  if (flag) {
    FI_CUDA(cudaMemset(c->err, 0, sizeof(int)), "clear error flag");
    return fail(FI_E_TIMEOUT, "a bounded device-side wait gave up; results of the last calls are invalid");
  }
  return FI_OK;
}

}  // namespace

extern "C" {

const char* fi_status_str(fi_status s) {
  switch (s) {
    case FI_OK: return "ok";
    case FI_E_INVALID: return "invalid argument";
    case FI_E_OOM: return "out of device memory";
    case FI_E_CUDA: return "CUDA error";
    case FI_E_STATE: return "invalid state";
    case FI_E_TIMEOUT: return "device wait timed out";
    case FI_E_UNSUPPORTED: return "unsupported";
  }
  return "unknown status";
}

const char* fi_last_error(void) { return g_last_error.c_str(); }

fi_status fi_init(fi_ctx** out, const fi_config* cfg, const void* h, void* stream) {
  if (!out) return fail(FI_E_INVALID, "out is NULL");
  *out = nullptr;
  if (!cfg || !h) return fail(FI_E_INVALID, "cfg or h is NULL");
  for (int k = 0; k < 4; ++k)
    if (cfg->reserved[k] != 0) return fail(FI_E_INVALID, "reserved fields must be 0");
  if (cfg->tc_max != 0 && cfg->tc_max != -1 && (!pow2(cfg->tc_max) || cfg->tc_max < (1 << kMinFftLog2)))
    return fail(FI_E_INVALID, "tc_max must be 0, -1 or a power of two >= 64");
  if (cfg->layers < 1 || cfg->channels < 1 || cfg->batch < 1) return fail(FI_E_INVALID, "layers, channels, batch must be >= 1");
  if (!pow2(cfg->max_len) || cfg->max_len < 2 || cfg->max_len > (1 << 17))
    return fail(FI_E_INVALID, "max_len must be a power of two in [2, 2^17]");
  if (cfg->dtype != FI_F32 && cfg->dtype != FI_BF16) return fail(FI_E_INVALID, "dtype must be FI_F32 or FI_BF16");
  if (cfg->chunk != 0 && (!pow2(cfg->chunk) || cfg->chunk < 2 || cfg->chunk > 64))
    return fail(FI_E_INVALID, "chunk must be 0 or a power of two in [2, 64]");
  if (cfg->fft_from != 0 && (!pow2(cfg->fft_from) || cfg->fft_from < (1 << kMinFftLog2)))
    return fail(FI_E_INVALID, "fft_from must be 0 or a power of two >= 64");
  const int64_t S = (int64_t)cfg->batch * cfg->channels;
  if (S > (1 << 24) || (int64_t)cfg->layers * cfg->channels > (1 << 24) || cfg->layers > 4096)
    return fail(FI_E_UNSUPPORTED, "too many streams or layers");

  fi_ctx* c = new (std::nothrow) fi_ctx();
  if (!c) return fail(FI_E_OOM, "host allocation failed");
  c->cfg = *cfg;
  c->st = reinterpret_cast<cudaStream_t>(stream);
  Dims& g = c->g;
  g.M = cfg->layers;
  g.D = cfg->channels;
  g.L = cfg->max_len;
  g.B = cfg->batch;
  g.S = (int)S;
  g.P = ilog2((uint32_t)g.L);
  g.bf16 = cfg->dtype == FI_BF16;

  auto bail = [&](fi_status s) { free_ctx(c); return s; };
  cudaError_t e;
  if ((e = cudaGetDevice(&c->device)) != cudaSuccess) return bail(cuda_fail(e, "cudaGetDevice"));
  int v = 0;
  if ((e = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, c->device)) != cudaSuccess)
    return bail(cuda_fail(e, "cudaDeviceGetAttribute"));
  c->num_sms = v;
  if ((e = cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, c->device)) != cudaSuccess)
    return bail(cuda_fail(e, "cudaDeviceGetAttribute"));
  c->max_smem = (size_t)v;

  // Plan: blocks below `chunk` on chip, FFT from `fft_from` up to the largest
  // transform one CTA holds, direct blocks from HBM in between and above.
  c->chunk = cfg->chunk ? cfg->chunk : 64;
  if (c->chunk > g.L) c->chunk = g.L;
  // FFT blocks pay off once a launch has enough (layer, stream) rows to fill the
  // GPU; tiny stacks keep direct blocks up to side 512.
  c->fft_from = cfg->fft_from ? cfg->fft_from : ((int64_t)g.M * g.S >= 2048 ? 64 : 1024);
  c->q_lo = ilog2((uint32_t)c->fft_from);
  c->q_hi = g.P - 1 < kMaxFftLog2 ? g.P - 1 : kMaxFftLog2;
  if (c->q_lo < kMinFftLog2) c->q_lo = kMinFftLog2;
  // Tensor-core blocks from side 64 up to tc_max, ahead of FFT (the FFT range
  // starts above them). Automatic: bf16 batches of 32 or more sequences, sides
  // 64..256 (64..512 from B = 64), where they measured faster than the FFT
  // blocks on B200 (8 x 2048 channels, L = 16384: B = 32 378 vs 391 ms per
  // generation, B = 64 748 vs 779 ms; B = 8 and fp32 B = 4 stay on FFT);
  // sides that cannot be planned are left to FFT.
  const bool tc_auto = cfg->tc_max == 0 && g.bf16 && g.B >= 32;
  if (cfg->tc_max > 0 || tc_auto) {
    c->tc_q_hi = ilog2((uint32_t)(tc_auto ? (g.B >= 64 ? 512 : 256) : cfg->tc_max));
    if (c->tc_q_hi > g.P - 1) c->tc_q_hi = g.P - 1;
    for (int q = kMinFftLog2; q <= c->tc_q_hi; ++q) {
      if ((e = tc_prepare(g, 1 << q, g.bf16 ? 0 : 1, c->num_sms, &c->tc[q])) != cudaSuccess) {
        if (tc_auto) {
          c->tc_q_hi = q - 1;
          break;
        }
        return bail(fail(FI_E_UNSUPPORTED, std::string("tensor-core blocks of side ") + std::to_string(1 << q) +
                                               " cannot be planned for this batch: " + cudaGetErrorString(e)));
      }
    }
    if (c->tc_q_hi >= kMinFftLog2 && c->q_lo <= c->tc_q_hi) c->q_lo = c->tc_q_hi + 1;
    if (c->tc_q_hi < kMinFftLog2) c->tc_q_hi = -1;
  }
  c->chunk_G = chunk_streams_per_cta(g, c->chunk, c->num_sms, c->max_smem);
  if (c->chunk_G == 0) return bail(fail(FI_E_UNSUPPORTED, "too many layers for the on-chip chunk window"));
  // Measured: an FFT grid launched early settles wherever it finds room and
  // runs slower there, on SMs a small chunk grid leaves idle (B = 1 stacks)
  // or beside chunk CTAs that leave registers free (short stacks). So only
  // chunk grids of whole-SM CTAs that leave at most a sixteenth of the SMs
  // idle take it.
  c->pdl_blocks = chunk_cta_fills_sm(g, c->chunk_G) &&
                  (g.S + c->chunk_G - 1) / c->chunk_G >= c->num_sms - c->num_sms / 16;
  if ((e = configure_chunk(chunk_smem_bytes(g, c->chunk, c->chunk_G))) != cudaSuccess)
    return bail(cuda_fail(e, "configure chunk kernel"));

  fi_status s;
  const size_t state_n = (size_t)(g.M + 1) * g.S * g.L;
  if ((s = dev_alloc((void**)&c->state, state_n * sizeof(float), "state")) != FI_OK) return bail(s);
  const size_t taps_n = (size_t)g.M * g.D * g.L;
  if ((s = dev_alloc((void**)&c->taps, taps_n * sizeof(float), "filters")) != FI_OK) return bail(s);
  size_t spec_n = 0;
  for (int q = c->q_lo; q <= c->q_hi; ++q) {
    c->spec_off[q] = spec_n;
    spec_n += (size_t)g.M * g.D * ((size_t(1) << q) + 1);
  }
  // Blocks wider than the largest transform: 2m-1 segment spectra per level.
  const int q_part_hi = c->q_lo <= kMaxFftLog2 ? g.P - 1 : -1;
  int m_max = 0;
  for (int q = kMaxFftLog2 + 1; q <= q_part_hi; ++q) {
    const int m = 1 << (q - kMaxFftLog2);
    c->spec_off[q] = spec_n;
    spec_n += (size_t)g.M * g.D * (2 * m - 1) * ((size_t(1) << kMaxFftLog2) + 1);
    m_max = m;
  }
  if (spec_n && (s = dev_alloc((void**)&c->spectra, spec_n * sizeof(float2), "spectra")) != FI_OK) return bail(s);
  if ((s = dev_alloc((void**)&c->twiddle, (size_t)kTwiddleN * sizeof(float2), "twiddles")) != FI_OK) return bail(s);
  if (m_max > 0 &&
      (s = dev_alloc((void**)&c->part_xs, (size_t)g.M * g.S * m_max * ((size_t(1) << kMaxFftLog2) + 1) * sizeof(float2),
                     "wide-block spectra")) != FI_OK)
    return bail(s);
  if ((s = dev_alloc((void**)&c->err, sizeof(int), "error flag")) != FI_OK) return bail(s);
  if ((e = cudaMemsetAsync(c->err, 0, sizeof(int), c->st)) != cudaSuccess) return bail(cuda_fail(e, "error flag"));

  std::vector<float2> tw(kTwiddleN);
  for (int m = 0; m < kTwiddleN; ++m) {
    const double ang = 2.0 * M_PI * (double)m / (double)kTwiddleN;
    tw[m] = make_float2((float)std::cos(ang), (float)(-std::sin(ang)));
  }
  if ((e = cudaMemcpyAsync(c->twiddle, tw.data(), tw.size() * sizeof(float2), cudaMemcpyHostToDevice, c->st)) != cudaSuccess)
    return bail(cuda_fail(e, "twiddle upload"));
  if ((e = launch_widen_filters(h, g.bf16, taps_n, c->taps, c->st)) != cudaSuccess) return bail(cuda_fail(e, "filter copy"));
  for (int q = c->q_lo; q <= c->q_hi; ++q)
    if ((e = launch_spectra(g, c->taps, c->spectra + c->spec_off[q], c->twiddle, q, c->st)) != cudaSuccess)
      return bail(cuda_fail(e, "spectra precompute"));
  for (int q = kMaxFftLog2 + 1; q <= q_part_hi; ++q)
    if ((e = launch_part_spectra(g, c->taps, c->spectra + c->spec_off[q], c->twiddle, 1 << (q - kMaxFftLog2), c->st)) !=
        cudaSuccess)
      return bail(cuda_fail(e, "wide-block spectra precompute"));
  if ((e = cudaStreamSynchronize(c->st)) != cudaSuccess) return bail(cuda_fail(e, "fi_init synchronize"));
  *out = c;
  return FI_OK;
}

fi_status fi_destroy(fi_ctx* c) {
  if (!c) return FI_OK;
  cudaStreamSynchronize(c->st);
  free_ctx(c);
  return FI_OK;
}

fi_status fi_reset(fi_ctx* c) {
  if (!c) return fail(FI_E_INVALID, "ctx is NULL");
  c->pos = 0;
  c->lazy_mode = 0;
  return FI_OK;
}

fi_status fi_set_mlp_block(fi_ctx* c, int32_t hidden, const float* w1, const float* b1, const float* w2,
                           const float* b2) {
  if (!c) return fail(FI_E_INVALID, "ctx is NULL");
  if (c->pos != 0 || c->lazy_mode) return fail(FI_E_STATE, "the block can change at position 0 only (call fi_reset)");
  if (hidden < 0) return fail(FI_E_INVALID, "hidden < 0");
  if (hidden > 0 && (!w1 || !b1 || !w2 || !b2)) return fail(FI_E_INVALID, "NULL weight");
  if (hidden > 0 && mlp_smem_bytes(c->g, hidden) > c->max_smem)
    return fail(FI_E_UNSUPPORTED, "channels or hidden width beyond one CTA's shared memory");
  // a captured position of an earlier fi_generate may still be in flight
  FI_CUDA(cudaStreamSynchronize(c->st), "synchronize");
  free_mlp(c);
  if (hidden == 0) return FI_OK;
  MlpBlock& m = c->mlp;
  const size_t M = c->g.M, D = c->g.D, H = hidden, B = c->g.B;
  fi_status s;
  if ((s = dev_alloc((void**)&m.w1, M * H * D * sizeof(float), "block weights")) != FI_OK ||
      (s = dev_alloc((void**)&m.b1, M * H * sizeof(float), "block biases")) != FI_OK ||
      (s = dev_alloc((void**)&m.w2, M * D * H * sizeof(float), "block weights")) != FI_OK ||
      (s = dev_alloc((void**)&m.b2, M * D * sizeof(float), "block biases")) != FI_OK ||
      (s = dev_alloc((void**)&m.z, B * H * sizeof(float), "block scratch")) != FI_OK ||
      (s = dev_alloc((void**)&m.y, B * D * sizeof(float), "block scratch")) != FI_OK ||
      (s = dev_alloc((void**)&m.pos, sizeof(MlpPos), "block position")) != FI_OK) {
    free_mlp(c);
    return s;
  }
  m.hidden = hidden;
  FI_CUDA(prepare_mlp(c->g, m), "block shared memory limit");
  FI_CUDA(cudaMemcpyAsync(m.w1, w1, M * H * D * sizeof(float), cudaMemcpyDeviceToDevice, c->st), "copy block weights");
  FI_CUDA(cudaMemcpyAsync(m.b1, b1, M * H * sizeof(float), cudaMemcpyDeviceToDevice, c->st), "copy block biases");
  FI_CUDA(cudaMemcpyAsync(m.w2, w2, M * D * H * sizeof(float), cudaMemcpyDeviceToDevice, c->st), "copy block weights");
  FI_CUDA(cudaMemcpyAsync(m.b2, b2, M * D * sizeof(float), cudaMemcpyDeviceToDevice, c->st), "copy block biases");
  return FI_OK;
}

fi_status fi_position(const fi_ctx* c, int32_t* pos) {
  if (!c || !pos) return fail(FI_E_INVALID, "NULL argument");
  *pos = c->pos;
  return FI_OK;
}

fi_status fi_set_stream(fi_ctx* c, void* stream) {
  if (!c) return fail(FI_E_INVALID, "ctx is NULL");
  c->st = reinterpret_cast<cudaStream_t>(stream);
  return FI_OK;
}

fi_status fi_get_plan(const fi_ctx* c, int32_t* chunk, int32_t* fft_from, int32_t* tc_max) {
  if (!c) return fail(FI_E_INVALID, "ctx is NULL");
  if (chunk) *chunk = c->chunk;
  if (fft_from) *fft_from = c->q_lo <= c->q_hi ? (1 << c->q_lo) : 0;
  if (tc_max) *tc_max = c->tc_q_hi >= kMinFftLog2 ? (1 << c->tc_q_hi) : 0;
  return FI_OK;
}

// The channel-mixing block's launches of one position as a graph: the small
// block of step t, then every layer's two launches, all reading the position
// record *mlp.pos, and a last node that advances it,
// so one instantiation serves every position of every fi_generate call (the
// per-call record is written by a launch before the first position). Captured
// once per fi_set_mlp_block, on a stream of the context's own.
fi_status mlp_layers_graph(fi_ctx* c) {
  if (c->mlp_graph) return FI_OK;
  if (!c->cap_st) FI_CUDA(cudaStreamCreateWithFlags(&c->cap_st, cudaStreamNonBlocking), "capture stream");
  FI_CUDA(cudaStreamBeginCapture(c->cap_st, cudaStreamCaptureModeThreadLocal), "begin capture");
  cudaError_t e = cudaSuccess;
  const MlpPos unused{};
  e = launch_mlp_block(c->g, c->state, c->taps, unused, c->mlp.pos, c->mlp.y, c->cap_st);
  for (int l = 1; l <= c->g.M && e == cudaSuccess; ++l)
    e = launch_mlp_layer(c->g, c->state, c->taps, c->mlp, l, unused, c->mlp.pos, c->cap_st);
  if (e == cudaSuccess) e = launch_mlp_next(c->mlp.pos, c->cap_st);
  cudaGraph_t graph = nullptr;
  const cudaError_t e_end = cudaStreamEndCapture(c->cap_st, &graph);
  if (e == cudaSuccess) e = e_end;
  if (e == cudaSuccess) e = cudaGraphInstantiate(&c->mlp_graph, graph, 0);
  if (graph) cudaGraphDestroy(graph);
  if (e != cudaSuccess) {
    cudaGetLastError();
    c->mlp_graph = nullptr;
    return fail(FI_E_CUDA, std::string("capturing the block's layers: ") + cudaGetErrorString(e));
  }
  return FI_OK;
}

// One position with the channel-mixing block: the token (x_t may be NULL: it
// is already in the state), the block of step t (from HBM when wider than
// kMlpBlockMax, else in the position's own launches), then per layer the
// block's products (after the last layer, with noise, the sampler). graph:
// those launches run as one launch of the captured graph, at the position
// *mlp.pos holds (set to p before the first position).
fi_status mlp_position(fi_ctx* c, const MlpPos& p, const void* x_t, bool graph) {
  fi_status s;
  const int t = p.t;
  if (x_t && (s = timed(c, KC_TOKEN, [&] { return launch_mlp_token(c->g, c->state, x_t, t, c->st); },
                        "token store")) != FI_OK)
    return s;
  // blocks wider than kMlpBlockMax from HBM first; narrower ones run in the position's launches
  if (t >= 1 && lowbit(t) > kMlpBlockMax && (s = run_block(c, t)) != FI_OK) return s;
  if (graph)
    return timed(c, KC_TOKEN, [&] { return cudaGraphLaunch(c->mlp_graph, c->st); }, "block graph launch", -1,
                 2 * c->g.M + 2);
  if ((s = timed(c, KC_TOKEN, [&] { return launch_mlp_block(c->g, c->state, c->taps, p, nullptr, c->mlp.y, c->st); },
                 "small block launch")) != FI_OK)
    return s;
  for (int l = 1; l <= c->g.M; ++l)
    if ((s = timed(c, KC_TOKEN, [&] { return launch_mlp_layer(c->g, c->state, c->taps, c->mlp, l, p, nullptr, c->st); },
                   "channel-mixing block launch", -1, 2)) != FI_OK)
      return s;
  return FI_OK;
}

fi_status fi_step(fi_ctx* c, const void* x_t, float* y_t) {
  if (!c || !x_t || !y_t) return fail(FI_E_INVALID, "NULL argument");
  if (c->pos >= c->g.L) return fail(FI_E_STATE, "position == max_len");
  if (c->lazy_mode) return fail(FI_E_STATE, "context holds a lazy generation; call fi_reset");
  fi_status s;
  const int t = c->pos;
  if (c->mlp.hidden > 0) {
    const MlpPos p{t, t, 1, 0.f, nullptr, y_t, nullptr};
    if ((s = mlp_position(c, p, x_t, false)) != FI_OK) return s;
    c->pos++;
    return FI_OK;
  }
  // small blocks (direct, side <= kTokenBlockMax) run inside the red-cell launch
  const int fused_u = (t >= 1 && token_block_fused(c->g, lowbit(t))) ? lowbit(t) : 0;
  if (t >= 1 && !fused_u && (s = run_block(c, t)) != FI_OK) return s;
  if ((s = timed(c, KC_TOKEN,
                 [&] { return launch_token(c->g, c->state, c->taps, t, x_t, nullptr, 0.f, y_t, c->st, fused_u); },
                 "red-cell launch")) != FI_OK)
    return s;
  c->pos++;
  return FI_OK;
}

fi_status fi_generate(fi_ctx* c, int32_t n, const void* x0, const float* eps, float eps_scale, float* y_out,
                      float* rec) {
  if (!c) return fail(FI_E_INVALID, "ctx is NULL");
  if (n < 0) return fail(FI_E_INVALID, "n < 0");
  if (n == 0) return FI_OK;
  if (!eps || !y_out) return fail(FI_E_INVALID, "NULL buffer");
  if (!x0 && c->pos == 0) return fail(FI_E_INVALID, "x0 may be NULL only when continuing from a position > 0");
  if ((int64_t)c->pos + n > c->g.L) return fail(FI_E_STATE, "position + n > max_len");
  if (c->lazy_mode) return fail(FI_E_STATE, "context holds a lazy generation; call fi_reset");
  const int CH = c->chunk;
  const int base = c->pos, end = c->pos + n;
  int p = base;
  fi_status s;
  if (c->mlp.hidden > 0) {
    // one position alone runs its launches directly; more replay the captured layers
    const bool graph = n >= 2;
    const MlpPos p0{base, base, n, eps_scale, eps, y_out, rec};
    if (graph) {
      if ((s = mlp_layers_graph(c)) != FI_OK) return s;
      if ((s = timed(c, KC_TOKEN, [&] { return launch_mlp_set(c->mlp.pos, p0, c->st); }, "block position")) != FI_OK)
        return s;
    }
    for (int t = base; t < end; ++t) {
      MlpPos p = p0;
      p.t = t;
      if ((s = mlp_position(c, p, t == base ? x0 : nullptr, graph)) != FI_OK) return s;
    }
    c->pos = end;
    return FI_OK;
  }
  while (p < end) {
    const int cst = (p / CH) * CH;
    const int p1 = (cst + CH < end) ? cst + CH : end;
    int last_done = p - 1;
    if (p == cst && cst > 0) {
      if ((s = run_block(c, cst)) != FI_OK) return s;
      last_done = cst;
    }
    ChunkArgs a{};
    a.state = c->state;
    a.taps = c->taps;
    a.x0 = (p == base) ? x0 : nullptr;
    a.eps = eps;
    a.eps_scale = eps_scale;
    a.y_out = y_out;
    a.rec = rec;
    a.n_gen = n;
    a.gen_base = base;
    a.c = cst;
    a.chunk = CH;
    a.p0 = p;
    a.p1 = p1;
    a.last_done = last_done;
    a.err = c->err;
    a.wait_limit = c->wait_limit;
    a.trigger = c->pdl_blocks ? 1 : 0;
    if ((s = timed(c, KC_CHUNK, [&] { return launch_chunk(c->g, a, c->chunk_G, c->st); }, "chunk launch")) != FI_OK)
      return s;
    p = p1;
  }
  c->pos = end;
  return FI_OK;
}

fi_status fi_prefill(fi_ctx* c, int32_t p, const void* x, float* y_out, float* rec) {
  if (!c || !x) return fail(FI_E_INVALID, "NULL argument");
  if (c->mlp.hidden > 0) return fail(FI_E_UNSUPPORTED, "prefill with the channel-mixing block is not supported");
  if (p < 1 || p > c->g.L) return fail(FI_E_INVALID, "p must be in [1, max_len]");
  if (p > (1 << kMaxFftLog2))
    return fail(FI_E_UNSUPPORTED, "prompts longer than " + std::to_string(1 << kMaxFftLog2) + " positions");
  if (c->pos != 0) return fail(FI_E_STATE, "fi_prefill starts a sequence: call fi_reset first");
  if (c->lazy_mode) return fail(FI_E_STATE, "context holds a lazy generation; call fi_reset");
  const Dims& g = c->g;
  const int q = prefix_transform_log2(p);
  const size_t need = (size_t)g.M * g.D * ((size_t(1) << q) + 1);
  if (need > c->pf_spec_n) {
    FI_CUDA(cudaStreamSynchronize(c->st), "synchronize");
    cudaFree(c->pf_spec);
    c->pf_spec = nullptr;
    c->pf_spec_n = 0;
    fi_status s = dev_alloc((void**)&c->pf_spec, need * sizeof(float2), "prefill spectra");
    if (s != FI_OK) return s;
    c->pf_spec_n = need;
  }
  fi_status s = timed(c, KC_FFT,
                      [&] { return launch_prefix(g, c->state, c->taps, c->pf_spec, c->twiddle, p, x, y_out, rec, c->st); },
                      "prefill launch");
  if (s != FI_OK) return s;
  // Blocks of steps i < p whose targets reach past the prompt (i + lowbit(i) > p):
  // their parts at targets >= p are what p calls of fi_step would have added
  // there. Increasing steps, so the first block to reach a target (a power-of-two
  // step) stores before the others add.
  for (int i = 1; i < p; ++i)
    if (i + (i & -i) > p && (s = run_block(c, i, p)) != FI_OK) return s;
  c->pos = p;
  return FI_OK;
}

fi_status fi_generate_host(fi_ctx* c, int32_t n, const void* x0_host, const float* eps_host, float eps_scale,
                           float* y_out_host) {
  if (!c) return fail(FI_E_INVALID, "ctx is NULL");
  if (n < 0) return fail(FI_E_INVALID, "n < 0");
  if (n == 0) return FI_OK;
  if (!x0_host || !eps_host || !y_out_host) return fail(FI_E_INVALID, "NULL buffer");
  if ((int64_t)c->pos + n > c->g.L) return fail(FI_E_STATE, "position + n > max_len");
  const size_t row = (size_t)c->g.S;
  const size_t esz = c->g.bf16 ? 2 : 4;
  if ((size_t)n > c->stage_n) {
    cudaFree(c->d_x0);
    cudaFree(c->d_eps);
    cudaFree(c->d_y);
    c->d_x0 = nullptr;
    c->d_eps = c->d_y = nullptr;
    c->stage_n = 0;
    fi_status s;
    if ((s = dev_alloc(&c->d_x0, row * 4, "staging x0")) != FI_OK) return s;
    if ((s = dev_alloc((void**)&c->d_eps, row * n * sizeof(float), "staging eps")) != FI_OK) return s;
    if ((s = dev_alloc((void**)&c->d_y, row * n * sizeof(float), "staging y")) != FI_OK) return s;
    c->stage_n = (size_t)n;
  }
  // Segments of whole chunks: segment k's noise is uploaded on up_st, generated
  // on the context's stream once it has arrived, and its outputs are read back
  // on dn_st once generated, so the copies of one segment overlap the
  // generation of others (with pinned host buffers). The generation itself is
  // the same as one fi_generate call: each segment continues from the state
  // the previous one left.
  const int per = (n + kHostSegments - 1) / kHostSegments;
  const int seg = per <= kHostSegmentMin ? n : ((per + kChunkMaxSteps - 1) / kChunkMaxSteps) * kChunkMaxSteps;
  const int nseg = (n + seg - 1) / seg;
  if (!c->up_st) FI_CUDA(cudaStreamCreateWithFlags(&c->up_st, cudaStreamNonBlocking), "copy stream");
  if (!c->dn_st) FI_CUDA(cudaStreamCreateWithFlags(&c->dn_st, cudaStreamNonBlocking), "copy stream");
  while (c->seg_ev.size() < 2 * (size_t)nseg + 1) {
    cudaEvent_t e;
    FI_CUDA(cudaEventCreateWithFlags(&e, cudaEventDisableTiming), "cudaEventCreate");
    c->seg_ev.push_back(e);
  }
  // Once a copy is queued, no return may leave one in flight on the caller's
  // host buffers: every failure below waits for both copy streams first.
  auto quiesce = [&](fi_status s) {
    cudaStreamSynchronize(c->up_st);
    cudaStreamSynchronize(c->dn_st);
    return s;
  };
  auto check = [&](cudaError_t e, const char* what) { return e == cudaSuccess ? FI_OK : quiesce(cuda_fail(e, what)); };
  fi_status s;
  // the staging buffers may still be read or written by an earlier call's work
  if ((s = check(cudaEventRecord(c->seg_ev[2 * nseg], c->st), "cudaEventRecord")) != FI_OK ||
      (s = check(cudaStreamWaitEvent(c->up_st, c->seg_ev[2 * nseg], 0), "cudaStreamWaitEvent")) != FI_OK ||
      (s = check(cudaMemcpyAsync(c->d_x0, x0_host, row * esz, cudaMemcpyHostToDevice, c->up_st), "x0 upload")) != FI_OK)
    return s;
  for (int k = 0; k < nseg; ++k) {
    const size_t off = (size_t)k * seg * row, cnt = (size_t)std::min(seg, n - k * seg) * row;
    if ((s = check(cudaMemcpyAsync(c->d_eps + off, eps_host + off, cnt * sizeof(float), cudaMemcpyHostToDevice,
                                   c->up_st),
                   "eps upload")) != FI_OK ||
        (s = check(cudaEventRecord(c->seg_ev[2 * k], c->up_st), "cudaEventRecord")) != FI_OK)
      return s;
  }
  for (int k = 0; k < nseg; ++k) {
    const int nk = std::min(seg, n - k * seg);
    const size_t off = (size_t)k * seg * row;
    if ((s = check(cudaStreamWaitEvent(c->st, c->seg_ev[2 * k], 0), "cudaStreamWaitEvent")) != FI_OK) return s;
    if ((s = fi_generate(c, nk, k == 0 ? c->d_x0 : nullptr, c->d_eps + off, eps_scale, c->d_y + off, nullptr)) !=
        FI_OK)
      return quiesce(s);
    if ((s = check(cudaEventRecord(c->seg_ev[2 * k + 1], c->st), "cudaEventRecord")) != FI_OK ||
        (s = check(cudaStreamWaitEvent(c->dn_st, c->seg_ev[2 * k + 1], 0), "cudaStreamWaitEvent")) != FI_OK ||
        (s = check(cudaMemcpyAsync(y_out_host + off, c->d_y + off, (size_t)nk * row * sizeof(float),
                                   cudaMemcpyDeviceToHost, c->dn_st),
                   "y download")) != FI_OK)
      return s;
  }
  FI_CUDA(cudaStreamSynchronize(c->dn_st), "synchronize");
  return sync_and_check(c);
}

fi_status fi_sync(fi_ctx* c) {
  if (!c) return fail(FI_E_INVALID, "ctx is NULL");
  return sync_and_check(c);
}

fi_status fi_generate_lazy(fi_ctx* c, int32_t n, const void* x0, const float* eps, float eps_scale, float* y_out) {
  if (!c) return fail(FI_E_INVALID, "ctx is NULL");
  if (n < 0) return fail(FI_E_INVALID, "n < 0");
  if (n == 0) return FI_OK;
  if (!x0 || !eps || !y_out) return fail(FI_E_INVALID, "NULL buffer");
  if ((int64_t)c->pos + n > c->g.L) return fail(FI_E_STATE, "position + n > max_len");
  if (c->mlp.hidden > 0) return fail(FI_E_UNSUPPORTED, "the lazy baseline runs the elementwise block only");
  if (c->pos > 0 && !c->lazy_mode) return fail(FI_E_STATE, "context holds a relaxed generation; call fi_reset");
  c->lazy_mode = 1;
  const size_t row = (size_t)c->g.S;
  const int base = c->pos;
  fi_status s;
  for (int t = base; t < base + n; ++t) {
    if ((s = timed(c, KC_LAZY, [&] { return launch_lazy_sums(c->g, c->state, c->taps, t, c->st); }, "lazy launch")) !=
        FI_OK)
      return s;
    const void* xt = (t == base) ? x0 : nullptr;
    const float* et = eps + (size_t)(t - base) * row;
    float* yt = y_out + (size_t)(t - base) * row;
    if ((s = timed(c, KC_TOKEN, [&] { return launch_token(c->g, c->state, c->taps, t, xt, et, eps_scale, yt, c->st); },
                   "red-cell launch")) != FI_OK)
      return s;
  }
  c->pos = base + n;
  return FI_OK;
}

fi_status fi_read_activations(fi_ctx* c, int32_t layer, float* dst) {
  if (!c || !dst) return fail(FI_E_INVALID, "NULL argument");
  if (layer < 0 || layer >= c->g.M) return fail(FI_E_INVALID, "layer must be in [0, M-1]");
  FI_CUDA(launch_read_layer(c->g, c->state, layer, c->pos, dst, c->st), "read activations");
  return FI_OK;
}

fi_status fi_profile(fi_ctx* c, int32_t enable) {
  if (!c) return fail(FI_E_INVALID, "ctx is NULL");
  c->prof = enable ? 1 : 0;
  return FI_OK;
}

fi_status fi_profile_read(fi_ctx* c, int32_t counts[FI_NUM_KERNEL_CLASSES], double ms[FI_NUM_KERNEL_CLASSES]) {
  return fi_profile_read_sides(c, counts, ms, nullptr, nullptr);
}

fi_status fi_profile_read_sides(fi_ctx* c, int32_t counts[FI_NUM_KERNEL_CLASSES], double ms[FI_NUM_KERNEL_CLASSES],
                                int32_t side_counts[32], double side_ms[32]) {
  if (!c || !counts || !ms) return fail(FI_E_INVALID, "NULL argument");
  FI_CUDA(cudaStreamSynchronize(c->st), "profile synchronize");
  for (int k = 0; k < FI_NUM_KERNEL_CLASSES; ++k) {
    counts[k] = 0;
    ms[k] = 0.0;
  }
  for (int k = 0; k < 32; ++k) {
    if (side_counts) side_counts[k] = 0;
    if (side_ms) side_ms[k] = 0.0;
  }
  for (auto& e : c->ev_live) {
    float t = 0.f;
    FI_CUDA(cudaEventElapsedTime(&t, e.a, e.b), "cudaEventElapsedTime");
    counts[e.cls] += e.kernels;
    ms[e.cls] += t;
    if (e.side_q >= 0 && e.side_q < 32) {
      if (side_counts) side_counts[e.side_q] += 1;
      if (side_ms) side_ms[e.side_q] += t;
    }
    c->ev_free.push_back(e);
  }
  c->ev_live.clear();
  return FI_OK;
}

fi_status fi_debug_chunk_schedule(int32_t chunk, int32_t retimed, int32_t* out, int32_t cap, int32_t* count,
                                  int32_t* chain_lags) {
  if (!out || !count || cap < 0) return fail(FI_E_INVALID, "bad argument");
  if (!pow2(chunk) || chunk < 2 || chunk > kChunkMaxSteps) return fail(FI_E_INVALID, "chunk must be a power of two in [2, 64]");
  ChunkTable tab{};
  if (!build_chunk_table(chunk, retimed != 0, &tab, retimed == 2)) return fail(FI_E_UNSUPPORTED, "table too long");
  *count = tab.n;
  if (chain_lags) *chain_lags = tab.lag1;
  for (int j = 0; j < tab.n && j < cap; ++j) {
    const uint32_t e = tab.e[j];
    const int kind = (int)((e >> 21) & 15);
    out[5 * j + 0] = (int32_t)(e & 127);
    out[5 * j + 1] = (int32_t)((e >> 7) & 127);
    out[5 * j + 2] = chunk_piece_sources(kind);
    out[5 * j + 3] = (int32_t)((e >> 14) & 127);
    out[5 * j + 4] = chunk_piece_targets(kind);
  }
  for (int r = 0; r < chunk; ++r) {
    for (int j = tab.first[r]; j < tab.first[r + 1]; ++j)
      if ((int)(tab.e[j] & 127) != r) return fail(FI_E_STATE, "step index does not match the entries");
  }
  return FI_OK;
}

fi_status fi_debug_set_wait_limit(fi_ctx* c, int32_t limit) {
  if (!c) return fail(FI_E_INVALID, "ctx is NULL");
  c->wait_limit = limit < 0 ? kDefaultWaitLimit : limit;
  return FI_OK;
}

fi_status fi_debug_fft(int32_t log2n, int32_t count, const float* in, float* out, int32_t inverse, void* stream) {
  if (!in || !out || count < 0) return fail(FI_E_INVALID, "bad argument");
  if (log2n < kMinFftLog2 || log2n > kMaxFftLog2) return fail(FI_E_INVALID, "log2n must be in [6, 14]");
  if (count == 0) return FI_OK;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  std::vector<float2> tw(kTwiddleN);
  for (int m = 0; m < kTwiddleN; ++m) {
    const double ang = 2.0 * M_PI * (double)m / (double)kTwiddleN;
    tw[m] = make_float2((float)std::cos(ang), (float)(-std::sin(ang)));
  }
  float2* dtw = nullptr;
  fi_status s = dev_alloc((void**)&dtw, tw.size() * sizeof(float2), "twiddles");
  if (s != FI_OK) return s;
  cudaError_t e = cudaMemcpyAsync(dtw, tw.data(), tw.size() * sizeof(float2), cudaMemcpyHostToDevice, st);
  if (e == cudaSuccess)
    e = launch_debug_fft(log2n, count, reinterpret_cast<const float2*>(in), reinterpret_cast<float2*>(out), inverse,
                         dtw, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  cudaFree(dtw);
  if (e != cudaSuccess) return cuda_fail(e, "debug FFT");
  return FI_OK;
}

}  // extern "C"
