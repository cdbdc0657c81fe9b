// Channel-mixing block: the Flash Inference summary page's synthetic setting
// ("Configurazione Sperimentale": the blocks are MLP + GELU, the sampler adds
// noise; "Architettura del Modello": block^l maps R^D to R^D). Read as one
// hidden layer of width Dh per layer:
//   a^l_t = R(W2^l GELU(W1^l y^l_t + b1^l) + b2^l)   (per sequence b, across channels),
// with y^l_t = acc^l_t + h^l_0 a^{l-1}_t (the red cell) and GELU(u) = u Phi(u)
// (the exact form, from erff). Unlike tanh the block mixes channels, so layer
// l+1 at position t needs every channel of layer l at t: each position runs,
// per layer, one launch for the red cells and the first product (every CTA
// forms the y it needs in shared memory) and one for the second product, which
// writes the activations back into the state slots (or, after the last layer,
// the sampler's next token).
#include "fi_internal.cuh"

namespace fi {

namespace {

constexpr int kMlpThreads = 256;               // 8 warps, one output row per warp at a time
constexpr int kMlpRowsPerCta = 32;

__device__ __forceinline__ float gelu_exact(float u) { return 0.5f * u * (1.0f + erff(u * 0.70710678118654752f)); }

// Dot product of a weight row (length n, contiguous) with the vector in shared
// memory, by one warp: lanes stride the row, then a shuffle reduction.
__device__ __forceinline__ float warp_dot(const float* __restrict__ w, const float* v, int n, int lane) {
  float sum = 0.f;
  for (int k = lane; k < n; k += 32) sum = fmaf(__ldg(w + k), v[k], sum);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  return sum;
}

// Red cells of layer l at position t for sequence b (all D channels, into
// shared memory), then z[b][k] = GELU(W1[k] . y + b1[k]) for this CTA's rows k.
// The first CTA of each sequence also writes y^l_t to rec (and to y_out for the
// last layer). grid = (ceil(Dh / kMlpRowsPerCta), B).
__global__ void __launch_bounds__(kMlpThreads) k_mlp_in(Dims g, const float* __restrict__ state,
                                                       const float* __restrict__ taps, int l, int t, int hidden,
                                                       const float* __restrict__ w1, const float* __restrict__ b1,
                                                       float* __restrict__ z, float* __restrict__ y_out,
                                                       float* __restrict__ rec, int n_gen, int gen_base) {
  extern __shared__ float ysm[];   // [D]
  const int b = blockIdx.y;
  for (int d = threadIdx.x; d < g.D; d += blockDim.x) {
    const int s = d * g.B + b;
    const float acc = t == 0 ? 0.f : state[slot_index(g, l, s, t)];
    const float a_in = state[slot_index(g, l - 1, s, t)];
    const float y = fmaf(taps[((size_t)(l - 1) * g.D + d) * g.L], a_in, acc);
    ysm[d] = y;
    if (blockIdx.x == 0) {
      const size_t io = (size_t)b * g.D + d;
      if (rec) rec[((size_t)(l - 1) * n_gen + (t - gen_base)) * g.S + io] = y;
      if (y_out && l == g.M) y_out[(size_t)(t - gen_base) * g.S + io] = y;
    }
  }
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* W1 = w1 + (size_t)(l - 1) * hidden * g.D;
  const int k_hi = min(hidden, (int)(blockIdx.x + 1) * kMlpRowsPerCta);
  for (int k = blockIdx.x * kMlpRowsPerCta + warp; k < k_hi; k += kMlpThreads / 32) {
    const float u = warp_dot(W1 + (size_t)k * g.D, ysm, g.D, lane) + b1[(size_t)(l - 1) * hidden + k];
    if (lane == 0) z[(size_t)b * hidden + k] = gelu_exact(u);
  }
}

// a[d] = W2[d] . z_b + b2[d] for this CTA's channels d; stored as the
// activation a^l_t (l < M), or, after the last layer and with noise given, as
// the next token x_{t+1} = R(a + eps_scale eps_t). grid = (ceil(D / kMlpRowsPerCta), B).
__global__ void __launch_bounds__(kMlpThreads) k_mlp_out(Dims g, float* __restrict__ state, int l, int t, int hidden,
                                                        const float* __restrict__ w2, const float* __restrict__ b2,
                                                        const float* __restrict__ z, const float* __restrict__ eps_t,
                                                        float eps_scale) {
  extern __shared__ float zsm[];   // [hidden]
  const int b = blockIdx.y;
  for (int k = threadIdx.x; k < hidden; k += blockDim.x) zsm[k] = z[(size_t)b * hidden + k];
  __syncthreads();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const float* W2 = w2 + (size_t)(l - 1) * g.D * hidden;
  const int d_hi = min(g.D, (int)(blockIdx.x + 1) * kMlpRowsPerCta);
  for (int d = blockIdx.x * kMlpRowsPerCta + warp; d < d_hi; d += kMlpThreads / 32) {
    const float a = warp_dot(W2 + (size_t)d * hidden, zsm, hidden, lane) + b2[(size_t)(l - 1) * g.D + d];
    if (lane != 0) continue;
    const int s = d * g.B + b;
    if (l < g.M) {
      state[slot_index(g, l, s, t)] = round_act(a, g.bf16);
    } else if (eps_t && t + 1 < g.L) {
      state[slot_index(g, 0, s, t + 1)] = round_act(a + eps_scale * eps_t[(size_t)b * g.D + d], g.bf16);
    }
  }
}

// Token x_t [B][D] (context dtype) into slot (0, s, t), rounded as the state holds it.
__global__ void k_mlp_token(Dims g, float* __restrict__ state, const void* __restrict__ x, int t) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= g.S) return;
  const int b = i / g.D, d = i - b * g.D;
  state[slot_index(g, 0, d * g.B + b, t)] = round_act(load_token(x, (size_t)i, g.bf16), g.bf16);
}

}  // namespace

cudaError_t launch_mlp_token(const Dims& g, float* state, const void* x, int t, cudaStream_t st) {
  k_mlp_token<<<(g.S + 255) / 256, 256, 0, st>>>(g, state, x, t);
  return cudaGetLastError();
}

cudaError_t launch_mlp_layer(const Dims& g, float* state, const float* taps, const MlpBlock& m, int l, int t,
                             const float* eps_t, float eps_scale, float* y_out, float* rec, int n_gen, int gen_base,
                             cudaStream_t st) {
  const size_t smem_in = (size_t)g.D * sizeof(float), smem_out = (size_t)m.hidden * sizeof(float);
  if (smem_in > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_mlp_in, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_in);
    if (e != cudaSuccess) return e;
  }
  if (smem_out > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_mlp_out, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_out);
    if (e != cudaSuccess) return e;
  }
  const dim3 grid_in((unsigned)((m.hidden + kMlpRowsPerCta - 1) / kMlpRowsPerCta), (unsigned)g.B);
  k_mlp_in<<<grid_in, kMlpThreads, smem_in, st>>>(g, state, taps, l, t, m.hidden, m.w1, m.b1, m.z, y_out, rec, n_gen,
                                                  gen_base);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const dim3 grid_out((unsigned)((g.D + kMlpRowsPerCta - 1) / kMlpRowsPerCta), (unsigned)g.B);
  k_mlp_out<<<grid_out, kMlpThreads, smem_out, st>>>(g, state, l, t, m.hidden, m.w2, m.b2, m.z, eps_t, eps_scale);
  return cudaGetLastError();
}

}  // namespace fi
