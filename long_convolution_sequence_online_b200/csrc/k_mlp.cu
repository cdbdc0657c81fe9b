// Channel-mixing block: the Flash Inference summary page's synthetic setting
// ("Configurazione Sperimentale": the blocks are MLP + GELU, the sampler adds
// noise; "Architettura del Modello": block^l maps R^D to R^D). Read as one
// hidden layer of width Dh per layer:
//   a^l_t = R(W2^l GELU(W1^l y^l_t + b1^l) + b2^l)   (per sequence b, across channels),
// with y^l_t = acc^l_t + h^l_0 a^{l-1}_t (the red cell) and GELU(u) = u Phi(u)
// (the exact form, from erff). Unlike tanh the block mixes channels, so layer
// l+1 at position t needs every channel of layer l at t. Each position runs one
// launch for the schedule's small block of step t and layer 1's red cells,
// then per layer one launch for the first product and one for the second.
//
// Both products are matrix-vector work on weights that stay in L2 (a few MB
// per layer), so they are latency-bound: one warp owns one weight row, its
// lanes load the row as independent float4s, and every row is applied to up to
// kMlpGroup sequences at once (the row is read once per group, not once per
// sequence). The second product also forms the next layer's red cell y^{l+1}_t
// for its channel into a dense [B][D] buffer, so no launch gathers a layer's
// inputs from the strided state. Launches are programmatic: each loads what
// does not depend on the launch before it (weights, biases, taps, and for the
// second product the next accumulator and the noise) before it waits.
#include <mutex>
#include <type_traits>

#include "fi_internal.cuh"

namespace fi {

namespace {

constexpr int kMlpThreads = 256;   // 8 warps, one weight row each
constexpr int kMlpRows = kMlpThreads / 32;

__device__ __forceinline__ float gelu_exact(float u) { return 0.5f * u * (1.0f + erff(u * 0.70710678118654752f)); }

// A weight row held by one warp: the first kMlpPre float4s per lane are
// loaded before the kernel waits for the launch before it (they do not depend
// on it), the rest of a longer row is streamed in dots().
constexpr int kMlpPre = 8;
struct WarpRow {
  float4 w[kMlpPre];

  __device__ __forceinline__ void preload(const float* __restrict__ row, int n, int lane) {
    const float4* w4 = reinterpret_cast<const float4*>(row);
    const int n4 = (n & 3) == 0 ? n >> 2 : 0;
#pragma unroll
    for (int u = 0; u < kMlpPre; ++u) {
      const int c = lane + 32 * u;
      w[u] = c < n4 ? __ldg(w4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }

  // acc[b] = row . v[b] over n for b < nb (all lanes get the sums); v: nb
  // vectors of length n in shared memory, stride n.
  __device__ __forceinline__ void dots(const float* __restrict__ row, const float* v, int n, int nb, int lane,
                                       float (&acc)[kMlpGroup]) const {
#pragma unroll
    for (int b = 0; b < kMlpGroup; ++b) acc[b] = 0.f;
    if ((n & 3) == 0) {
      const int n4 = n >> 2;
#pragma unroll
      for (int u = 0; u < kMlpPre; ++u) {
        const int c = lane + 32 * u;
        if (c >= n4) break;
        add4(w[u], v, n, c, nb, acc);
      }
      const float4* w4 = reinterpret_cast<const float4*>(row);
      for (int c0 = lane + 32 * kMlpPre; c0 < n4; c0 += 4 * 32) {
        float4 wv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + 32 * u;
          wv[u] = c < n4 ? __ldg(w4 + c) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int c = c0 + 32 * u;
          if (c >= n4) break;
          add4(wv[u], v, n, c, nb, acc);
        }
      }
    } else {
      for (int k = lane; k < n; k += 32) {
        const float wk = __ldg(row + k);
#pragma unroll
        for (int b = 0; b < kMlpGroup; ++b) {
          if (b >= nb) break;
          acc[b] = fmaf(wk, v[(size_t)b * n + k], acc[b]);
        }
      }
    }
#pragma unroll
    for (int b = 0; b < kMlpGroup; ++b) {
      if (b >= nb) break;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[b] += __shfl_xor_sync(0xffffffffu, acc[b], o);
    }
  }

  static __device__ __forceinline__ void add4(const float4& wv, const float* v, int n, int c, int nb,
                                              float (&acc)[kMlpGroup]) {
#pragma unroll
    for (int b = 0; b < kMlpGroup; ++b) {
      if (b >= nb) break;
      const float4 x = *reinterpret_cast<const float4*>(v + (size_t)b * n + 4 * c);
      acc[b] = fmaf(wv.x, x.x, acc[b]);
      acc[b] = fmaf(wv.y, x.y, acc[b]);
      acc[b] = fmaf(wv.z, x.z, acc[b]);
      acc[b] = fmaf(wv.w, x.w, acc[b]);
    }
  }
};

// Where y^l_t goes besides the block's input: rec [M][n_gen][B][D] and, for
// the last layer, y_out [n_gen][B][D].
__device__ __forceinline__ void record_y(const Dims& g, int l, const MlpPos& p, int b, int d, float y) {
  const size_t io = (size_t)b * g.D + d;
  if (p.rec) p.rec[((size_t)(l - 1) * p.n_gen + (p.t - p.gen_base)) * g.S + io] = y;
  if (p.y_out && l == g.M) p.y_out[(size_t)(p.t - p.gen_base) * g.S + io] = y;
}

// z[b][k] = GELU(W1[k] . y_b + b1[k]) for the CTA's rows k and its group of
// sequences, y_b the layer's red cells in the dense ybuf [B][D] (written by the
// launch before). grid = (ceil(Dh / kMlpRows), ceil(B / kMlpGroup)).
__global__ void __launch_bounds__(kMlpThreads) k_mlp_in(Dims g, int l, int hidden, const float* __restrict__ w1,
                                                       const float* __restrict__ b1, const float* __restrict__ ybuf,
                                                       float* __restrict__ z) {
  extern __shared__ __align__(16) float ysm[];   // [nb][D]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = blockIdx.x * kMlpRows + warp;
  const float* row = w1 + ((size_t)(l - 1) * hidden + (k < hidden ? k : 0)) * g.D;
  WarpRow wr;
  wr.preload(row, k < hidden ? g.D : 0, lane);
  const float bias = k < hidden ? __ldg(b1 + (size_t)(l - 1) * hidden + k) : 0.f;
  pdl_wait_primary();   // ybuf comes from the launch before
  pdl_launch_dependents();
  const int b0 = blockIdx.y * kMlpGroup, nb = min(kMlpGroup, g.B - b0);
  const int n_in = nb * g.D;
  for (int i = threadIdx.x; i < n_in; i += blockDim.x) ysm[i] = ybuf[(size_t)b0 * g.D + i];
  __syncthreads();
  if (k >= hidden) return;
  float acc[kMlpGroup];
  wr.dots(row, ysm, g.D, nb, lane, acc);
#pragma unroll
  for (int b = 0; b < kMlpGroup; ++b)
    if (b < nb && lane == b) z[(size_t)(b0 + b) * hidden + k] = gelu_exact(acc[b] + bias);
}

// a[b][d] = W2[d] . z_b + b2[d] for the CTA's channels d. Layers l < M store
// R(a) as the activation a^l_t and form the next red cell
// y^{l+1}_t = acc^{l+1}_t + h^{l+1}_0 R(a) into ybuf; the last layer, with
// noise given, stores the next token x_{t+1} = R(a + eps_scale eps_t).
// grid = (ceil(D / kMlpRows), ceil(B / kMlpGroup)).
__global__ void __launch_bounds__(kMlpThreads) k_mlp_out(Dims g, float* __restrict__ state,
                                                        const float* __restrict__ taps, int l, MlpPos p_host,
                                                        const MlpPos* __restrict__ p_dev, int hidden,
                                                        const float* __restrict__ w2, const float* __restrict__ b2,
                                                        const float* __restrict__ z, float* __restrict__ ybuf) {
  extern __shared__ __align__(16) float zsm[];   // [nb][hidden]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = blockIdx.x * kMlpRows + warp;
  const float* row = w2 + ((size_t)(l - 1) * g.D + (d < g.D ? d : 0)) * hidden;
  WarpRow wr;
  wr.preload(row, d < g.D ? hidden : 0, lane);
  const float bias = d < g.D ? __ldg(b2 + (size_t)(l - 1) * g.D + d) : 0.f;
  const float h0 = l < g.M && d < g.D ? __ldg(taps + ((size_t)l * g.D + d) * g.L) : 0.f;
  const MlpPos p = p_dev ? *p_dev : p_host;
  const int t = p.t;
  const int b0 = blockIdx.y * kMlpGroup, nb = min(kMlpGroup, g.B - b0);
  // Launches trigger their dependents only after their own wait, so every
  // launch before the previous one has completed here: the next layer's
  // accumulator at t (final once the small block ran) and the noise can be read
  // before waiting.
  float acc_next = 0.f, e = 0.f;
  if (d < g.D && lane < nb) {
    const int s = d * g.B + b0 + lane;
    if (l < g.M && t > 0) acc_next = state[slot_index(g, l + 1, s, t)];
    if (l == g.M && p.eps && t + 1 < g.L) e = p.eps[(size_t)(t - p.gen_base) * g.S + (size_t)(b0 + lane) * g.D + d];
  }
  pdl_wait_primary();   // z comes from the launch before
  pdl_launch_dependents();
  for (int i = threadIdx.x; i < nb * hidden; i += blockDim.x) zsm[i] = z[(size_t)b0 * hidden + i];
  __syncthreads();
  if (d >= g.D) return;
  float acc[kMlpGroup];
  wr.dots(row, zsm, hidden, nb, lane, acc);
  float a = 0.f;
#pragma unroll
  for (int b = 0; b < kMlpGroup; ++b)
    if (lane == b) a = acc[b] + bias;
  if (lane >= nb) return;
  const int b = b0 + lane, s = d * g.B + b;
  if (l < g.M) {
    const float a_r = round_act(a, g.bf16);
    state[slot_index(g, l, s, t)] = a_r;
    const float y = fmaf(h0, a_r, acc_next);
    ybuf[(size_t)b * g.D + d] = y;
    record_y(g, l + 1, p, b, d, y);
  } else if (p.eps && t + 1 < g.L) {
    state[slot_index(g, 0, s, t + 1)] = round_act(a + p.eps_scale * e, g.bf16);
  }
}

// The block of step t, side UB = lowbit(t) <= kMlpBlockMax, for layer l and
// stream s (channel d): slot(l, s, t+u') (+)= sum_{u<UB} h^l[UB+u'-u]
// a^{l-1}_{t-UB+u}, stored when t is a power of two (the first block to reach
// these targets). Sources, targets and taps are read as vectors: t is a
// multiple of UB and every row of the state and taps starts 16-byte aligned.
template <int UB>
__device__ __forceinline__ float small_block(const Dims& g, float* __restrict__ state, const float* __restrict__ taps,
                                            int t, int l, int s, int d) {
  constexpr int V = UB >= 4 ? 4 : UB;   // floats per vector access
  using vec = typename std::conditional<V == 4, float4, typename std::conditional<V == 2, float2, float>::type>::type;
  float x[UB], h[2 * UB], cur[UB];
  const float* xp = state + slot_index(g, l - 1, s, t - UB);
  float* dp = state + slot_index(g, l, s, t);
  const float* hp = taps + ((size_t)(l - 1) * g.D + d) * g.L;
#pragma unroll
  for (int u = 0; u < UB; u += V) *reinterpret_cast<vec*>(x + u) = *reinterpret_cast<const vec*>(xp + u);
  if constexpr (V == 1) {
    *reinterpret_cast<float2*>(h) = __ldg(reinterpret_cast<const float2*>(hp));
  } else {
#pragma unroll
    for (int k = 0; k < 2 * UB; k += V) *reinterpret_cast<vec*>(h + k) = __ldg(reinterpret_cast<const vec*>(hp + k));
  }
  if (t == UB) {
#pragma unroll
    for (int up = 0; up < UB; ++up) cur[up] = 0.f;
  } else {
#pragma unroll
    for (int up = 0; up < UB; up += V) *reinterpret_cast<vec*>(cur + up) = *reinterpret_cast<const vec*>(dp + up);
  }
#pragma unroll
  for (int up = 0; up < UB; ++up) {
#pragma unroll
    for (int u = 0; u < UB; ++u) cur[up] = fmaf(h[UB + up - u], x[u], cur[up]);
  }
#pragma unroll
  for (int up = 0; up < UB; up += V) *reinterpret_cast<vec*>(dp + up) = *reinterpret_cast<const vec*>(cur + up);
  return cur[0];
}

// The position's small block for every (layer, stream), one thread each (a
// no-op at t = 0 and where lowbit(t) > kMlpBlockMax: that block ran before,
// from HBM); the layer-1 threads then form the red cell
// y^1_t = acc^1_t + h^1_0 x_t into ybuf [B][D] (and the records), the first
// layer's input.
__global__ void k_mlp_block(Dims g, float* __restrict__ state, const float* __restrict__ taps, MlpPos p_host,
                            const MlpPos* __restrict__ p_dev, float* __restrict__ ybuf) {
  pdl_launch_dependents();   // the first layer's launch loads its weights meanwhile
  const MlpPos p = p_dev ? *p_dev : p_host;
  const int t = p.t;
  const int U = t & -t;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= g.M * g.S) return;
  const int l = i / g.S + 1, s = i - (l - 1) * g.S, d = s / g.B;
  float acc;
  if (t == 0) {
    acc = 0.f;
  } else {
    switch (U) {
      case 1: acc = small_block<1>(g, state, taps, t, l, s, d); break;
      case 2: acc = small_block<2>(g, state, taps, t, l, s, d); break;
      case 4: acc = small_block<4>(g, state, taps, t, l, s, d); break;
      case kMlpBlockMax: acc = small_block<kMlpBlockMax>(g, state, taps, t, l, s, d); break;
      default:   // the block ran before: only layer 1's accumulator is read here
        if (l != 1) return;
        acc = state[slot_index(g, 1, s, t)];
        break;
    }
  }
  if (l != 1) return;
  const int b = s - d * g.B;
  const float y = fmaf(__ldg(taps + (size_t)d * g.L), state[slot_index(g, 0, s, t)], acc);
  ybuf[(size_t)b * g.D + d] = y;
  record_y(g, 1, p, b, d, y);
}

// The position counter of a captured position: advanced once all its layers ran.
__global__ void k_mlp_next(MlpPos* p_dev) { p_dev->t += 1; }
__global__ void k_mlp_set(MlpPos* p_dev, MlpPos v) { *p_dev = v; }

// Token x_t [B][D] (context dtype) into slot (0, s, t), rounded as the state holds it.
__global__ void k_mlp_token(Dims g, float* __restrict__ state, const void* __restrict__ x, int t) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= g.S) return;
  const int b = i / g.D, d = i - b * g.D;
  state[slot_index(g, 0, d * g.B + b, t)] = round_act(load_token(x, (size_t)i, g.bf16), g.bf16);
}

size_t smem_in_bytes(const Dims& g) { return (size_t)(g.B < kMlpGroup ? g.B : kMlpGroup) * g.D * sizeof(float); }
size_t smem_out_bytes(const Dims& g, int hidden) {
  return (size_t)(g.B < kMlpGroup ? g.B : kMlpGroup) * hidden * sizeof(float);
}

}  // namespace

size_t mlp_smem_bytes(const Dims& g, int hidden) {
  const size_t a = smem_in_bytes(g), b = smem_out_bytes(g, hidden);
  return a > b ? a : b;
}

cudaError_t launch_mlp_token(const Dims& g, float* state, const void* x, int t, cudaStream_t st) {
  k_mlp_token<<<(g.S + 255) / 256, 256, 0, st>>>(g, state, x, t);
  return cudaGetLastError();
}

// The dynamic shared-memory cap is one value per kernel for the whole process:
// raise it when this shape needs more, never lower it (another context may
// need more).
template <class K>
static cudaError_t raise_cap(K kernel, size_t smem) {
  if (smem <= 48 * 1024) return cudaSuccess;
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  cudaFuncAttributes fa{};
  cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
  if (e != cudaSuccess) return e;
  if ((size_t)fa.maxDynamicSharedSizeBytes >= smem) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

cudaError_t prepare_mlp(const Dims& g, const MlpBlock& m) {
  cudaError_t e = raise_cap(k_mlp_in, smem_in_bytes(g));
  if (e == cudaSuccess) e = raise_cap(k_mlp_out, smem_out_bytes(g, m.hidden));
  return e;
}

// Both launches allow programmatic stream serialization: each kernel may start
// while the launch before it drains, loads its weight rows, then waits for it.
cudaError_t launch_mlp_layer(const Dims& g, float* state, const float* taps, const MlpBlock& m, int l,
                             const MlpPos& p, const MlpPos* p_dev, cudaStream_t st) {
  const unsigned groups = (unsigned)((g.B + kMlpGroup - 1) / kMlpGroup);
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kMlpThreads);
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cfg.gridDim = dim3((unsigned)((m.hidden + kMlpRows - 1) / kMlpRows), groups);
  cfg.dynamicSmemBytes = smem_in_bytes(g);
  cudaError_t e = cudaLaunchKernelEx(&cfg, k_mlp_in, g, l, m.hidden, (const float*)m.w1, (const float*)m.b1,
                                     (const float*)m.y, m.z);
  if (e != cudaSuccess) return e;
  cfg.gridDim = dim3((unsigned)((g.D + kMlpRows - 1) / kMlpRows), groups);
  cfg.dynamicSmemBytes = smem_out_bytes(g, m.hidden);
  return cudaLaunchKernelEx(&cfg, k_mlp_out, g, state, taps, l, p, p_dev, m.hidden, (const float*)m.w2,
                            (const float*)m.b2, (const float*)m.z, m.y);
}

cudaError_t launch_mlp_block(const Dims& g, float* state, const float* taps, const MlpPos& p, const MlpPos* p_dev,
                             float* ybuf, cudaStream_t st) {
  const int n = g.M * g.S;
  k_mlp_block<<<(n + 255) / 256, 256, 0, st>>>(g, state, taps, p, p_dev, ybuf);
  return cudaGetLastError();
}

cudaError_t launch_mlp_next(MlpPos* p_dev, cudaStream_t st) {
  k_mlp_next<<<1, 1, 0, st>>>(p_dev);
  return cudaGetLastError();
}

cudaError_t launch_mlp_set(MlpPos* p_dev, const MlpPos& v, cudaStream_t st) {
  k_mlp_set<<<1, 1, 0, st>>>(p_dev, v);
  return cudaGetLastError();
}

}  // namespace fi
