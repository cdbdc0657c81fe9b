// The on-chip part of the relaxed schedule.
//
// Split the positions into aligned chunks of C (a power of two). At a step i
// inside a chunk [c, c+C) (i != c) the block side U = lowbit(i) equals
// lowbit(i - c) < C, its sources [i-U, i) and targets [i, i+U) both lie inside
// the chunk (i - c is a multiple of U, and (i-c) + lowbit(i-c) <= C). So every
// block smaller than C reads and writes only the current chunk, and a CTA that
// owns a set of streams can keep that chunk of every layer's activations and
// accumulators in shared memory and run C positions without touching HBM:
// the small gray blocks (Algorithm 1), then the red cells and blocks layer by
// layer (Algorithm 2/3), then the sampler. Blocks of side >= C happen only at
// chunk starts and are launched before this kernel (direct or FFT, from HBM).
//
// Streams are independent (the block and sampler act elementwise), so CTAs
// never wait on each other.
#include "fi_internal.cuh"

namespace fi {

struct ChunkShape {
  int G, GdMax, CH, CHP;
  size_t win, tp, h0, ep, total;  // float offsets / total floats
};

__host__ __device__ inline ChunkShape chunk_shape(const Dims& g, int CH, int G) {
  ChunkShape c;
  c.G = G;
  c.CH = CH;
  c.CHP = CH + 1;                  // odd stride: per-stream rows fall in different banks
  c.GdMax = (G - 1) / g.B + 2;     // channels a run of G consecutive streams can touch
  c.win = 0;
  c.tp = c.win + (size_t)(g.M + 1) * G * c.CHP;
  c.h0 = c.tp + (size_t)g.M * c.GdMax * CH;
  c.ep = c.h0 + (size_t)g.M * c.GdMax;
  c.total = c.ep + (size_t)CH * G;
  return c;
}

__device__ __forceinline__ int highbit_dev(int t) { return 1 << (31 - __clz(t)); }

__global__ void __launch_bounds__(256) k_chunk(Dims g, ChunkArgs a, int G) {
  extern __shared__ float csm[];
  const ChunkShape cs = chunk_shape(g, a.chunk, G);
  const int CH = cs.CH, CHP = cs.CHP, GdMax = cs.GdMax;
  float* win = csm + cs.win;   // [(M+1)][G][CHP]   slot window of positions [c, c+CH)
  float* tp = csm + cs.tp;     // [M][GdMax][CH]    taps h[0..CH)
  float* h0s = csm + cs.h0;    // [M][GdMax]        h[0]
  float* ep = csm + cs.ep;     // [CH][G]           sampler noise
  const int s0 = blockIdx.x * G;
  const int Gc = min(G, g.S - s0);
  const int d_lo = s0 / g.B;
  const int Gd = (s0 + Gc - 1) / g.B - d_lo + 1;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int r0 = a.p0 - a.c, r1 = a.p1 - a.c;

  for (int k = tid; k < g.M * Gd * CH; k += nt) {
    const int j = k % CH, rest = k / CH, dl = rest % Gd, l = rest / Gd;
    const float v = a.taps[((size_t)l * g.D + d_lo + dl) * g.L + j];
    tp[(l * GdMax + dl) * CH + j] = v;
    if (j == 0) h0s[l * GdMax + dl] = v;
  }
  // Slots already in HBM: tokens and activations below p0; the token at p0 when
  // no x0 is given; accumulators that some block has reached (the first block to
  // reach position t runs at step highbit(t)). Everything else starts at 0.
  for (int k = tid; k < (g.M + 1) * Gc * CH; k += nt) {
    const int r = k % CH, rest = k / CH, gg = rest % Gc, l = rest / Gc;
    const int t = a.c + r;
    float v = 0.f;
    if (t < g.L) {
      bool valid = t < a.p0;
      if (l == 0) valid = valid || (t == a.p0 && a.x0 == nullptr);
      else valid = valid || (t >= 1 && highbit_dev(t) <= a.last_done);
      if (valid) v = a.state[slot_index(g, l, s0 + gg, t)];
    }
    win[(l * G + gg) * CHP + r] = v;
  }
  for (int k = tid; k < (r1 - r0) * Gc; k += nt) {
    const int gg = k % Gc, r = r0 + k / Gc;
    const int s = s0 + gg, d = s / g.B, b = s - d * g.B;
    ep[r * G + gg] = a.eps[(size_t)(a.c + r - a.gen_base) * g.S + (size_t)b * g.D + d];
  }
  if (a.x0 != nullptr && tid < Gc) {
    const int s = s0 + tid, d = s / g.B, b = s - d * g.B;
    win[tid * CHP + r0] = round_act(load_token(a.x0, (size_t)b * g.D + d, g.bf16), g.bf16);
  }
  __syncthreads();

  for (int r = r0; r < r1; ++r) {
    const int t = a.c + r;
    if (r > 0) {
      // Gray block of step t (side U < CH) for every layer and stream, on chip.
      const int U = r & -r;
      const int lu = __ffs(U) - 1;
      const int W = g.M * Gc * U;
      for (int w = tid; w < W; w += nt) {
        const int up = w & (U - 1);
        const int rest = w >> lu;
        const int gg = rest % Gc, l = rest / Gc + 1;
        const int dl = (s0 + gg) / g.B - d_lo;
        const float* hp = tp + ((l - 1) * GdMax + dl) * CH + U + up;
        const float* xp = win + ((l - 1) * G + gg) * CHP + r - U;
        float sum = 0.f;
        for (int u = 0; u < U; ++u) sum = fmaf(hp[-u], xp[u], sum);
        win[(l * G + gg) * CHP + r + up] += sum;
      }
      __syncthreads();
    }
    if (tid < Gc) {
      // Red cells and blocks through the layers, then the sampler.
      const int gg = tid, s = s0 + gg, d = s / g.B, b = s - d * g.B, dl = d - d_lo;
      const size_t io = (size_t)b * g.D + d;
      float av = win[gg * CHP + r];
      float y = 0.f;
      for (int l = 1; l <= g.M; ++l) {
        float* sp = win + (l * G + gg) * CHP + r;
        y = fmaf(h0s[(l - 1) * GdMax + dl], av, *sp);
        if (a.rec) a.rec[((size_t)(l - 1) * a.n_gen + (t - a.gen_base)) * g.S + io] = y;
        if (l < g.M) {
          av = round_act(tanhf(y), g.bf16);
          *sp = av;
        }
      }
      a.y_out[(size_t)(t - a.gen_base) * g.S + io] = y;
      if (t + 1 < g.L) {
        const float xn = round_act(tanhf(y) + a.eps_scale * ep[r * G + gg], g.bf16);
        if (r + 1 < CH) win[gg * CHP + r + 1] = xn;
        else a.state[slot_index(g, 0, s, t + 1)] = xn;
      }
    }
    __syncthreads();
  }

  // Write back positions [p0, c+CH): new tokens and activations below p1,
  // accumulators (including the small blocks' partial sums) from p1 on.
  const int nr = CH - r0;
  for (int k = tid; k < (g.M + 1) * Gc * nr; k += nt) {
    const int r = r0 + k % nr, rest = k / nr, gg = rest % Gc, l = rest / Gc;
    const int t = a.c + r;
    if (t < g.L) a.state[slot_index(g, l, s0 + gg, t)] = win[(l * G + gg) * CHP + r];
  }
}

size_t chunk_smem_bytes(const Dims& g, int chunk, int G) { return chunk_shape(g, chunk, G).total * sizeof(float); }

int chunk_streams_per_cta(const Dims& g, int chunk, int num_sms, size_t max_smem) {
  int G = (g.S + num_sms - 1) / num_sms;
  if (G > 256) G = 256;
  if (G < 1) G = 1;
  while (G > 1 && chunk_smem_bytes(g, chunk, G) > max_smem) G = (G + 1) / 2;
  if (chunk_smem_bytes(g, chunk, G) > max_smem) return 0;
  return G;
}

cudaError_t configure_chunk(size_t smem) {
  return cudaFuncSetAttribute(k_chunk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

cudaError_t launch_chunk(const Dims& g, const ChunkArgs& a, int G, cudaStream_t st) {
  const size_t smem = chunk_smem_bytes(g, a.chunk, G);
  const int blocks = (g.S + G - 1) / G;
  k_chunk<<<blocks, 256, smem, st>>>(g, a, G);
  return cudaGetLastError();
}

}  // namespace fi
