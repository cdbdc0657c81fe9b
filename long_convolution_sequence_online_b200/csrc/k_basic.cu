// Per-position red cells, direct blocks read from HBM, the Lazy method's sums
// and the layout conversions.
#include <mutex>
#include <type_traits>

#include "fi_internal.cuh"

namespace fi {

// ---------------------------------------------------------------------------
// Red cells and blocks of position t for every stream (Algorithm 2's per-layer
// loop: b^l_t += a^{l-1}_t h^l_0, a^l_t = R(tanh(b^l_t))). One thread carries one
// stream through all M layers, since each layer needs the previous one's output.
// x_t: token buffer [B][D] of the context dtype, or NULL to take the token
// already in slot (0, s, t). eps_t: NULL, or [B][D] noise for the sampler
// x_{t+1} = R(tanh(y^M_t) + eps_scale * eps_t), written to slot (0, s, t+1).
// ---------------------------------------------------------------------------
__global__ void k_token(Dims g, float* __restrict__ state, const float* __restrict__ taps, int t,
                        const void* __restrict__ x_t, const float* __restrict__ eps_t, float eps_scale,
                        float* __restrict__ y_t) {
  const int s = blockIdx.x * blockDim.x + threadIdx.x;
  if (s >= g.S) return;
  const int d = s / g.B, b = s - d * g.B;
  const size_t io = (size_t)b * g.D + d;
  float a;
  if (x_t) {
    a = round_act(load_token(x_t, io, g.bf16), g.bf16);
    state[slot_index(g, 0, s, t)] = a;
  } else {
    a = state[slot_index(g, 0, s, t)];
  }
  // The layers' accumulators and h_0 taps do not depend on the chain, so they are
  // loaded a group of layers at a time, all in flight together, before the group's
  // dependent red cells run.
  constexpr int kGroup = 8;
  float y = 0.f;
  for (int l0 = 1; l0 <= g.M; l0 += kGroup) {
    float acc[kGroup], h0[kGroup];
#pragma unroll
    for (int j = 0; j < kGroup; ++j) {
      const int l = l0 + j;
      acc[j] = 0.f;
      h0[j] = 0.f;
      if (l <= g.M) {
        if (t > 0) acc[j] = state[slot_index(g, l, s, t)];
        h0[j] = __ldg(taps + ((size_t)(l - 1) * g.D + d) * g.L);
      }
    }
#pragma unroll
    for (int j = 0; j < kGroup; ++j) {
      const int l = l0 + j;
      if (l > g.M) break;
      y = fmaf(h0[j], a, acc[j]);
      if (l < g.M) {
        a = round_act(tanhf(y), g.bf16);
        state[slot_index(g, l, s, t)] = a;
      }
    }
  }
  y_t[io] = y;
  if (eps_t && t + 1 < g.L) state[slot_index(g, 0, s, t + 1)] = round_act(tanhf(y) + eps_scale * eps_t[io], g.bf16);
}

// The same position with one thread per (stream, layer): a CTA holds 32 streams
// and all M layers (32*M threads), so every layer's accumulator, h_0 tap and
// (U > 0) direct block of step t are fetched and computed in parallel, and only
// the red-cell chain is serial (one warp, through shared memory). The block of
// step t, side U = lowbit(t), adds sum_{u<U} h^l[U+u'-u] a^{l-1}_{t-U+u} to the
// targets t+u' (u' < U) of layer l (stored, not added, when t is a power of two,
// the first block to reach them): target t's part goes straight into the chain,
// the others back to the state, as the direct block kernel would leave them.
template <int U>
__global__ void k_token_par(Dims g, float* __restrict__ state, const float* __restrict__ taps, int t,
                            const void* __restrict__ x_t, const float* __restrict__ eps_t, float eps_scale,
                            float* __restrict__ y_t) {
  extern __shared__ float tsm[];
  float* accs = tsm;               // [M][32] accumulator of (layer, lane) at t
  float* h0s = tsm + g.M * 32;     // [M][32] h^l_0 of the lane's channel
  const int lane = threadIdx.x & 31, li = threadIdx.x >> 5;
  const int s = blockIdx.x * 32 + lane;
  const bool ok = s < g.S;
  const int d = ok ? s / g.B : 0;
  const int b = s - d * g.B;
  const size_t io = (size_t)b * g.D + d;
  // The chain's token and noise depend on no layer's sum: read them first.
  float a_tok = 0.f, e = 0.f;
  if (li == 0 && ok) {
    a_tok = x_t ? round_act(load_token(x_t, io, g.bf16), g.bf16) : state[slot_index(g, 0, s, t)];
    if (eps_t && t + 1 < g.L) e = eps_t[io];
  }
  if (ok) {
    const int l = li + 1;
    const float* hp = taps + ((size_t)(l - 1) * g.D + d) * g.L;
    float* dp = state + slot_index(g, l, s, t);
    float acc;
    if constexpr (U == 0) {
      h0s[li * 32 + lane] = __ldg(hp);
      acc = (t == 0) ? 0.f : dp[0];
    } else {
      // Vector accesses: t is a multiple of U, and rows of the state and the
      // taps start 16-byte aligned (L >= 2U).
      constexpr int V = U >= 4 ? 4 : U;
      using vec = typename std::conditional<V == 4, float4, typename std::conditional<V == 2, float2, float>::type>::type;
      const bool overwrite = (t == U);   // lowbit(t) == t: t is a power of two
      const float* xp = state + slot_index(g, l - 1, s, t - U);
      float x[U], h[2 * U], cur[U];
#pragma unroll
      for (int u = 0; u < U; u += V) *reinterpret_cast<vec*>(x + u) = *reinterpret_cast<const vec*>(xp + u);
      if constexpr (V == 1) {
        *reinterpret_cast<float2*>(h) = __ldg(reinterpret_cast<const float2*>(hp));
      } else {
#pragma unroll
        for (int k = 0; k < 2 * U; k += V) *reinterpret_cast<vec*>(h + k) = __ldg(reinterpret_cast<const vec*>(hp + k));
      }
      if (overwrite) {
#pragma unroll
        for (int up = 0; up < U; ++up) cur[up] = 0.f;
      } else {
#pragma unroll
        for (int up = 0; up < U; up += V) *reinterpret_cast<vec*>(cur + up) = *reinterpret_cast<const vec*>(dp + up);
      }
#pragma unroll
      for (int up = 0; up < U; ++up) {
#pragma unroll
        for (int u = 0; u < U; ++u) cur[up] = fmaf(h[U + up - u], x[u], cur[up]);
      }
      h0s[li * 32 + lane] = h[0];
      acc = cur[0];
      // targets t+1 .. t+U-1 back to the state (slot t receives the red cell's
      // activation below, or for the last layer is not read again)
#pragma unroll
      for (int up = 0; up < U; up += V) *reinterpret_cast<vec*>(dp + up) = *reinterpret_cast<const vec*>(cur + up);
    }
    accs[li * 32 + lane] = acc;
  }
  __syncthreads();
  if (li != 0 || !ok) return;
  float a = a_tok;
  if (x_t) state[slot_index(g, 0, s, t)] = a;
  float y = 0.f;
  for (int l = 1; l <= g.M; ++l) {
    y = fmaf(h0s[(l - 1) * 32 + lane], a, accs[(l - 1) * 32 + lane]);
    if (l < g.M) {
      a = round_act(tanhf(y), g.bf16);
      state[slot_index(g, l, s, t)] = a;
    }
  }
  y_t[io] = y;
  if (eps_t && t + 1 < g.L) state[slot_index(g, 0, s, t + 1)] = round_act(tanhf(y) + eps_scale * e, g.bf16);
}

cudaError_t launch_token(const Dims& g, float* state, const float* taps, int t, const void* x_t,
                         const float* eps_t, float eps_scale, float* y_t, cudaStream_t st, int block_u) {
  if (g.M <= kTokenMaxLayers) {
    const unsigned blocks = (unsigned)((g.S + 31) / 32);
    const unsigned threads = 32u * (unsigned)g.M;
    const size_t smem = (size_t)2 * g.M * 32 * sizeof(float);
#define FI_TOKEN_PAR(UU) k_token_par<UU><<<blocks, threads, smem, st>>>(g, state, taps, t, x_t, eps_t, eps_scale, y_t)
    switch (block_u) {
      case 0: FI_TOKEN_PAR(0); break;
      case 1: FI_TOKEN_PAR(1); break;
      case 2: FI_TOKEN_PAR(2); break;
      case 4: FI_TOKEN_PAR(4); break;
      case kTokenBlockMax: FI_TOKEN_PAR(kTokenBlockMax); break;
      default: return cudaErrorInvalidValue;
    }
#undef FI_TOKEN_PAR
    return cudaGetLastError();
  }
  if (block_u != 0) return cudaErrorInvalidValue;
  const int threads = 128;
  k_token<<<(g.S + threads - 1) / threads, threads, 0, st>>>(g, state, taps, t, x_t, eps_t, eps_scale, y_t);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Direct block of step i, side U = lowbit(i) (the gray block of Algorithm 1 by
// its definition, tau(a, [i-U, i-1], h, [i, i+U-1])): for every layer l and
// stream s, slot(l, s, i+u') (+)= sum_{u<U} h^l[U+u'-u] * a^{l-1}[i-U+u].
// One CTA per (layer, channel, sequence); the 2U-1 taps and U sources are
// staged in shared memory. The block at a power-of-two step is the first to
// reach its targets and stores instead of adding.
// ---------------------------------------------------------------------------
__global__ void k_tile_direct(Dims g, float* __restrict__ state, const float* __restrict__ taps, int i, int U,
                              int overwrite, int t_min) {
  pdl_launch_dependents();
  extern __shared__ float dsm[];
  float* hs = dsm;          // taps h[0..2U)
  float* xs = dsm + 2 * U;  // sources a[i-U..i)
  const long cta = blockIdx.x;          // ((l-1)*D + d)*B + b
  const int b = (int)(cta % g.B);
  const long ld = cta / g.B;
  const int d = (int)(ld % g.D);
  const int l = (int)(ld / g.D) + 1;
  const int s = d * g.B + b;
  const float* hp = taps + ((size_t)(l - 1) * g.D + d) * g.L;
  const float* xp = state + slot_index(g, l - 1, s, i - U);
  for (int j = threadIdx.x; j < 2 * U; j += blockDim.x) hs[j] = hp[j];
  for (int j = threadIdx.x; j < U; j += blockDim.x) xs[j] = xp[j];
  __syncthreads();
  float* dp = state + slot_index(g, l, s, i);
  for (int up = threadIdx.x; up < U; up += blockDim.x) {
    if (i + up < t_min) continue;
    float sum = 0.f;
    for (int u = 0; u < U; ++u) sum = fmaf(hs[U + up - u], xs[u], sum);
    dp[up] = overwrite ? sum : dp[up] + sum;
  }
}

// The same block for small sides (U <= 32, the blocks fi_step takes from HBM at
// most positions): one thread per (row, target), U threads per row, so a launch
// is a few waves of short threads instead of one CTA per row. Taps h[U+u'-u] are
// contiguous across a row's threads; its sources are the same for all of them.
// U is a template argument so that the whole sum unrolls and a thread issues
// all its loads before the first product.
template <int U>
__global__ void k_tile_direct_small(Dims g, float* __restrict__ state, const float* __restrict__ taps, int i,
                                    int overwrite, int t_min) {
  pdl_launch_dependents();
  constexpr int log2u = U >= 32 ? 5 : U >= 16 ? 4 : U >= 8 ? 3 : U >= 4 ? 2 : U >= 2 ? 1 : 0;
  const long gid = (long)blockIdx.x * blockDim.x + threadIdx.x;
  const long row = gid >> log2u;        // ((l-1)*D + d)*B + b
  if (row >= (long)g.M * g.S) return;
  const int up = (int)(gid & (U - 1));
  if (i + up < t_min) return;
  const int b = (int)(row % g.B);
  const long ld = row / g.B;
  const int d = (int)(ld % g.D);
  const int l = (int)(ld / g.D) + 1;
  const int s = d * g.B + b;
  const float* hp = taps + ((size_t)(l - 1) * g.D + d) * g.L + U + up;
  const float* xp = state + slot_index(g, l - 1, s, i - U);
  float hv[U], xv[U];
#pragma unroll
  for (int u = 0; u < U; ++u) {
    hv[u] = __ldg(hp - u);
    xv[u] = __ldg(xp + u);
  }
  float sum = 0.f;
#pragma unroll
  for (int u = 0; u < U; ++u) sum = fmaf(hv[u], xv[u], sum);
  float* dp = state + slot_index(g, l, s, i + up);
  *dp = overwrite ? sum : *dp + sum;
}

// The same block for sides whose taps and sources do not fit in shared memory:
// taps and sources are read through the cache (every thread of the CTA reads the
// same source at the same time, and neighbouring threads neighbouring taps).
__global__ void k_tile_direct_big(Dims g, float* __restrict__ state, const float* __restrict__ taps, int i, int U,
                                  int overwrite, int t_min) {
  pdl_launch_dependents();
  const long cta = blockIdx.x;          // ((l-1)*D + d)*B + b
  const int b = (int)(cta % g.B);
  const long ld = cta / g.B;
  const int d = (int)(ld % g.D);
  const int l = (int)(ld / g.D) + 1;
  const int s = d * g.B + b;
  const float* hp = taps + ((size_t)(l - 1) * g.D + d) * g.L;
  const float* xp = state + slot_index(g, l - 1, s, i - U);
  float* dp = state + slot_index(g, l, s, i);
  for (int up = threadIdx.x; up < U; up += blockDim.x) {
    if (i + up < t_min) continue;
    float sum = 0.f;
    for (int u = 0; u < U; ++u) sum = fmaf(__ldg(hp + U + up - u), __ldg(xp + u), sum);
    dp[up] = overwrite ? sum : dp[up] + sum;
  }
}

cudaError_t launch_tile_direct(const Dims& g, float* state, const float* taps, int i, int t_min, cudaStream_t st) {
  const int U = i & -i;
  const long blocks_big = (long)g.M * g.D * g.B;
  if (U > 8192) {
    k_tile_direct_big<<<(unsigned)blocks_big, 256, 0, st>>>(g, state, taps, i, U, is_pow2(i) ? 1 : 0, t_min);
    return cudaGetLastError();
  }
  if (U <= 32) {
    const long threads_total = (long)g.M * g.S * U;
    const int threads = 256;
    const unsigned blocks = (unsigned)((threads_total + threads - 1) / threads);
    const int ow = is_pow2(i) ? 1 : 0;
    switch (U) {
      case 1: k_tile_direct_small<1><<<blocks, threads, 0, st>>>(g, state, taps, i, ow, t_min); break;
      case 2: k_tile_direct_small<2><<<blocks, threads, 0, st>>>(g, state, taps, i, ow, t_min); break;
      case 4: k_tile_direct_small<4><<<blocks, threads, 0, st>>>(g, state, taps, i, ow, t_min); break;
      case 8: k_tile_direct_small<8><<<blocks, threads, 0, st>>>(g, state, taps, i, ow, t_min); break;
      case 16: k_tile_direct_small<16><<<blocks, threads, 0, st>>>(g, state, taps, i, ow, t_min); break;
      default: k_tile_direct_small<32><<<blocks, threads, 0, st>>>(g, state, taps, i, ow, t_min); break;
    }
    return cudaGetLastError();
  }
  const size_t smem = (size_t)3 * U * sizeof(float);
  if (smem > 48 * 1024) {
    // one cap per kernel for the whole process: raise it, never lower it
    // (another context's launch may need more)
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    cudaFuncAttributes fa{};
    cudaError_t e = cudaFuncGetAttributes(&fa, k_tile_direct);
    if (e == cudaSuccess && (size_t)fa.maxDynamicSharedSizeBytes < smem)
      e = cudaFuncSetAttribute(k_tile_direct, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  const long blocks = (long)g.M * g.D * g.B;
  const int threads = U >= 256 ? 256 : (U < 32 ? 32 : U);
  k_tile_direct<<<(unsigned)blocks, threads, smem, st>>>(g, state, taps, i, U, is_pow2(i) ? 1 : 0, t_min);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// The Lazy method's sum for position t (summary page, "Tre Strategie di
// Calcolo", Metodo Lazy), all layers in one launch: slot(l, s, t) =
// sum_{s' < t} h^l[t-s'] a^{l-1}[s']. One warp per (layer, channel, group of up
// to 4 sequences), so each tap is read once per group.
// ---------------------------------------------------------------------------
__global__ void k_lazy(Dims g, float* __restrict__ state, const float* __restrict__ taps, int t) {
  const long warp = ((long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const int nbg = (g.B + 3) / 4;
  if (warp >= (long)g.M * g.D * nbg) return;
  const int bg = (int)(warp % nbg);
  const long ld = warp / nbg;
  const int d = (int)(ld % g.D);
  const int l = (int)(ld / g.D) + 1;
  const int b0 = bg * 4, nb = min(4, g.B - b0);
  const float* hp = taps + ((size_t)(l - 1) * g.D + d) * g.L;
  const float* xp[4];
  for (int j = 0; j < 4; ++j) xp[j] = state + slot_index(g, l - 1, d * g.B + b0 + min(j, nb - 1), 0);
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int sp = lane; sp < t; sp += 32) {
    const float h = hp[t - sp];
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j] = fmaf(h, xp[j][sp], acc[j]);
  }
#pragma unroll
  for (int j = 0; j < 4; ++j)
    for (int o = 16; o > 0; o >>= 1) acc[j] += __shfl_xor_sync(0xffffffffu, acc[j], o);
  if (lane < nb) {
    float v = acc[0];
#pragma unroll
    for (int j = 1; j < 4; ++j) v = (lane == j) ? acc[j] : v;
    state[slot_index(g, l, d * g.B + b0 + lane, t)] = v;
  }
}

cudaError_t launch_lazy_sums(const Dims& g, float* state, const float* taps, int t, cudaStream_t st) {
  const long warps = (long)g.M * g.D * ((g.B + 3) / 4);
  const int threads = 256;
  const long blocks = (warps * 32 + threads - 1) / threads;
  k_lazy<<<(unsigned)blocks, threads, 0, st>>>(g, state, taps, t);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Layout conversions.
// ---------------------------------------------------------------------------
__global__ void k_widen(const void* __restrict__ h, int bf16, size_t n, float* __restrict__ out) {
  for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < n; k += (size_t)gridDim.x * blockDim.x)
    out[k] = load_token(h, k, bf16);
}

cudaError_t launch_widen_filters(const void* h, int bf16, size_t n, float* out, cudaStream_t st) {
  k_widen<<<148 * 8, 256, 0, st>>>(h, bf16, n, out);
  return cudaGetLastError();
}

// dst[t][b][d] = slot(layer, d*B+b, t) for t < pos.
__global__ void k_read_layer(Dims g, const float* __restrict__ state, int layer, int pos, float* __restrict__ dst) {
  const size_t total = (size_t)pos * g.S;
  for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < total; k += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(k / g.S);
    const int r = (int)(k - (size_t)t * g.S);  // r = b*D + d
    const int b = r / g.D, d = r - b * g.D;
    dst[k] = state[slot_index(g, layer, d * g.B + b, t)];
  }
}

cudaError_t launch_read_layer(const Dims& g, const float* state, int layer, int pos, float* dst, cudaStream_t st) {
  if (pos == 0) return cudaSuccess;
  k_read_layer<<<148 * 8, 256, 0, st>>>(g, state, layer, pos, dst);
  return cudaGetLastError();
}

}  // namespace fi
