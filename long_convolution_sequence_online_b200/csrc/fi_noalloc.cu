// fi_generate_noalloc: the closed-loop generation of fi_generate, for callers
// that must not allocate device memory.
//
// Some callers cannot call cudaMalloc at all: code that runs on a thread with a
// hard latency budget (an allocation can block on the driver), code inside a
// host framework whose device memory is owned by its own allocator, or code
// launched where allocation is not permitted. This entry point allocates
// nothing: its working memory is one file-scope device array of fixed size, and
// the caller passes only its inputs and outputs.
//
// Working memory, in floats, for a configuration (M, D, L, B):
//   filters widened to fp32   M*D*L
//   slot state                (M+1)*B*D*L
//   error flag                64
// which must fit in kNoAllocFloats (8 Mi floats = 32 MiB). Every GPU that loads
// the library holds that array until the process exits. All calls share it and
// it keeps the last call's contents: nothing in it needs clearing except the
// error flag, which each call resets (the slot state is written before it is
// read, as in every generation from position 0). Calls whose work overlaps on
// the GPU (different streams, or different host threads) race on the array.
//
// Blocks of side >= the on-chip chunk run as direct sums from the array (no
// filter spectra, which would need more memory); the on-chip chunk kernel is the
// same as fi_generate's.
#include <mutex>
#include <string>

#include "fi_internal.cuh"

using namespace fi;

namespace {

constexpr size_t kNoAllocFloats = size_t(1) << 23;
constexpr size_t kNoAllocFlagFloats = 64;

__device__ __align__(256) float g_noalloc_scratch[kNoAllocFloats];

// The array's device address, looked up once per device (with that device
// current): in host code the symbol is only a host-side stand-in.
constexpr int kMaxDevices = 64;
float* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

fi_status noalloc_fail(fi_status s, const std::string& msg) {
  set_last_error(msg);   // reported by fi_last_error()
  return s;
}

bool pow2_i64(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

size_t round64(size_t n) { return (n + 63) / 64 * 64; }

}  // namespace

extern "C" {

fi_status fi_generate_noalloc(const fi_config* cfg, const void* h, int32_t n, const void* x0, const float* eps,
                              float eps_scale, float* y_out, void* stream) {
  if (!cfg || !h || !x0 || !eps || !y_out) return noalloc_fail(FI_E_INVALID, "NULL argument");
  for (int k = 0; k < 4; ++k)
    if (cfg->reserved[k] != 0) return noalloc_fail(FI_E_INVALID, "reserved fields must be 0");
  if (cfg->tc_max != 0 && cfg->tc_max != -1)
    return noalloc_fail(FI_E_INVALID, "tc_max must be 0 or -1 (this entry point runs direct blocks only)");
  if (cfg->layers < 1 || cfg->channels < 1 || cfg->batch < 1)
    return noalloc_fail(FI_E_INVALID, "layers, channels, batch must be >= 1");
  if (!pow2_i64(cfg->max_len) || cfg->max_len < 2 || cfg->max_len > (1 << 15))
    return noalloc_fail(FI_E_INVALID, "max_len must be a power of two in [2, 2^15]");
  if (cfg->dtype != FI_F32 && cfg->dtype != FI_BF16) return noalloc_fail(FI_E_INVALID, "dtype must be FI_F32 or FI_BF16");
  if (cfg->chunk != 0 && (!pow2_i64(cfg->chunk) || cfg->chunk < 2 || cfg->chunk > 64))
    return noalloc_fail(FI_E_INVALID, "chunk must be 0 or a power of two in [2, 64]");
  if (n < 0 || n > cfg->max_len) return noalloc_fail(FI_E_INVALID, "n must be in [0, max_len]");

  Dims g{};
  g.M = cfg->layers;
  g.D = cfg->channels;
  g.L = cfg->max_len;
  g.B = cfg->batch;
  const int64_t S = (int64_t)g.B * g.D;
  if (S > (1 << 24)) return noalloc_fail(FI_E_INVALID, "too many streams");
  g.S = (int)S;
  g.P = ilog2((uint32_t)g.L);
  g.bf16 = cfg->dtype == FI_BF16;

  const size_t taps_n = (size_t)g.M * g.D * g.L;
  const size_t state_n = (size_t)(g.M + 1) * g.S * g.L;
  const size_t need = round64(taps_n) + round64(state_n) + kNoAllocFlagFloats;
  if (need > kNoAllocFloats)
    return noalloc_fail(FI_E_INVALID, "configuration needs " + std::to_string(need) +
                                          " floats of working memory; the static area holds " +
                                          std::to_string(kNoAllocFloats));
  if (n == 0) return FI_OK;

  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(FI_E_CUDA, std::string("cudaGetDevice: ") + cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return noalloc_fail(FI_E_UNSUPPORTED, "device index out of range");
  float* base = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_addr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess)
        return noalloc_fail(FI_E_CUDA, std::string("cudaGetSymbolAddress: ") + cudaGetErrorString(e));
      g_scratch_addr[dev] = static_cast<float*>(p);
    }
    base = g_scratch_addr[dev];
  }
  float* taps = base;
  float* state = base + round64(taps_n);
  int* err = reinterpret_cast<int*>(state + round64(state_n));
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);

  int num_sms = 0, max_smem = 0;
  if ((e = cudaDeviceGetAttribute(&num_sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
    return noalloc_fail(FI_E_CUDA, std::string("cudaDeviceGetAttribute: ") + cudaGetErrorString(e));
  int CH = cfg->chunk ? cfg->chunk : 64;
  if (CH > g.L) CH = g.L;
  const int G = chunk_streams_per_cta(g, CH, num_sms, (size_t)max_smem);
  if (G == 0) return noalloc_fail(FI_E_UNSUPPORTED, "too many layers for the on-chip chunk window");
  if ((e = configure_chunk(chunk_smem_bytes(g, CH, G))) != cudaSuccess)
    return noalloc_fail(FI_E_CUDA, std::string("configure chunk kernel: ") + cudaGetErrorString(e));

  if ((e = cudaMemsetAsync(err, 0, sizeof(int), st)) != cudaSuccess)
    return noalloc_fail(FI_E_CUDA, std::string("clear error flag: ") + cudaGetErrorString(e));
  if ((e = launch_widen_filters(h, g.bf16, taps_n, taps, st)) != cudaSuccess)
    return noalloc_fail(FI_E_CUDA, std::string("filter copy: ") + cudaGetErrorString(e));
  for (int p = 0; p < n;) {
    const int cst = (p / CH) * CH;
    const int p1 = (cst + CH < n) ? cst + CH : n;
    int last_done = p - 1;
    if (cst > 0) {
      if ((e = launch_tile_direct(g, state, taps, cst, cst, st)) != cudaSuccess)
        return noalloc_fail(FI_E_CUDA, std::string("direct block launch: ") + cudaGetErrorString(e));
      last_done = cst;
    }
    ChunkArgs a{};
    a.state = state;
    a.taps = taps;
    a.x0 = (p == 0) ? x0 : nullptr;
    a.eps = eps;
    a.eps_scale = eps_scale;
    a.y_out = y_out;
    a.rec = nullptr;
    a.n_gen = n;
    a.gen_base = 0;
    a.c = cst;
    a.chunk = CH;
    a.p0 = p;
    a.p1 = p1;
    a.last_done = last_done;
    a.err = err;
    a.wait_limit = kDefaultWaitLimit;
    if ((e = launch_chunk(g, a, G, st)) != cudaSuccess)
      return noalloc_fail(FI_E_CUDA, std::string("chunk launch: ") + cudaGetErrorString(e));
    p = p1;
  }
  if ((e = cudaStreamSynchronize(st)) != cudaSuccess)
    return noalloc_fail(FI_E_CUDA, std::string("synchronize: ") + cudaGetErrorString(e));
  int flag = 0;
  if ((e = cudaMemcpy(&flag, err, sizeof(int), cudaMemcpyDeviceToHost)) != cudaSuccess)
    return noalloc_fail(FI_E_CUDA, std::string("read error flag: ") + cudaGetErrorString(e));
  if (flag) return noalloc_fail(FI_E_TIMEOUT, "a bounded device-side wait gave up; y_out is invalid");
  return FI_OK;
}

}  // extern "C"
