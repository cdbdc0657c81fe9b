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
//
// Thread roles: thread k owns the (layer, stream) rows k, k+T, ... for the gray
// blocks (all U outputs of a row, with U sources and 2U-1 taps in registers);
// threads [0, G) each carry one stream through the layers for the red cells.
#include <mutex>

#include "fi_internal.cuh"

namespace fi {

constexpr int kChunkMaxThreads = 512;
constexpr int kChunkMaxStreams = 128;
constexpr int kSuspendHintNs = 1000;   // longest a suspended barrier check may last

struct ChunkShape {
  int G, GdMax, CH, CHP, TPS, CW, NG, K;
  size_t win, tp, h0, ep, ys, flags, total;  // float offsets / total floats
};

__host__ __device__ inline ChunkShape chunk_shape(const Dims& g, int CH, int G) {
  ChunkShape c;
  c.G = G;
  c.CH = CH;
  c.CHP = CH + 1;                  // odd strides: rows of different streams / channels fall in different banks
  c.TPS = CH + 1;
  c.CW = (G + 31) / 32;            // chain warps (one stream per lane)
  c.GdMax = (G - 1) / g.B + 2;     // channels a run of G consecutive streams can touch
  c.win = 0;
  c.tp = c.win + (size_t)(g.M + 1) * G * c.CHP;
  c.h0 = c.tp + (size_t)g.M * c.GdMax * c.TPS;
  c.ep = c.h0 + (size_t)g.M * c.GdMax;
  c.ys = c.ep + (size_t)CH * G;
  c.flags = (c.ys + (size_t)CH * G + 1) & ~(size_t)1;   // 8-byte aligned mbarriers
  c.NG = g.M >= 2 ? 2 : 1;                              // layer groups per position
  c.K = (g.M + c.NG - 1) / c.NG;                        // layers per group
  c.total = c.flags + 2 * (size_t)(2 * c.NG) * c.CW;    // act_ready[NG][CW] + tile_done[NG][CW]
  return c;
}

__device__ __forceinline__ int highbit_dev(int t) { return 1 << (31 - __clz(t)); }

// 4-byte asynchronous global -> shared copy; `valid` false writes 0 instead.
__device__ __forceinline__ void cp_async4(float* dst, const float* src, bool valid) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src), "r"(valid ? 4 : 0)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Gray block of side U for one (layer, stream) row: dst[r+u'] += sum_u h[U+u'-u] src[r-U+u].
// Outputs go in groups of OB; for a group the taps h[U+u'-u] form a window that
// slides by one per source u, so each step loads one source and one new tap and
// issues OB FMAs from registers.
template <int U>
__device__ __forceinline__ void small_block(const float* __restrict__ src, float* __restrict__ dst,
                                            const float* __restrict__ taps, int r) {
  constexpr int OB = U < 16 ? U : 16;
  const float* x = src + r - U;
#pragma unroll
  for (int up0 = 0; up0 < U; up0 += OB) {
    float acc[OB], w[OB];
#pragma unroll
    for (int k = 0; k < OB; ++k) {
      acc[k] = 0.f;
      w[k] = taps[U + up0 + k];          // tap of output up0+k for source u = 0
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const float xv = x[u];
#pragma unroll
      for (int k = 0; k < OB; ++k) acc[k] = fmaf(w[k], xv, acc[k]);
      if (u + 1 < U) {
#pragma unroll
        for (int k = OB - 1; k > 0; --k) w[k] = w[k - 1];
        w[0] = taps[U + up0 - u - 1];
      }
    }
#pragma unroll
    for (int k = 0; k < OB; ++k) dst[r + up0 + k] += acc[k];
  }
}

__device__ __forceinline__ void gray_block(int U, const float* src, float* dst, const float* taps, int r) {
  switch (U) {
    case 1: small_block<1>(src, dst, taps, r); break;
    case 2: small_block<2>(src, dst, taps, r); break;
    case 4: small_block<4>(src, dst, taps, r); break;
    case 8: small_block<8>(src, dst, taps, r); break;
    case 16: small_block<16>(src, dst, taps, r); break;
    default: small_block<32>(src, dst, taps, r); break;
  }
}

// tanh for the block and the sampler, without branches (every lane of the chain
// warp takes the same path).
// fp32 activations: two forms evaluated side by side and selected by |y|.
//  * |y| >= 0.55: tanh|y| = 1 - 2 / (1 + e^(2|y|)) with the hardware exp2 and
//    reciprocal, e^(2|y|) = 2^(2 |y| log2 e) (overflow to +inf gives exactly 1),
//    sign restored after. 2/(1+e) <= 0.5 here, so the subtraction loses nothing.
//  * |y| < 0.55: y * P(y^2), P a degree-5 polynomial fitted to tanh(y)/y by
//    weighted least squares on that interval (fit error 1e-9).
// Relative error within about 5e-7 for every y (1e-7 in the polynomial range).
// The polynomial runs in parallel with the exp2/reciprocal chain, so the
// critical path of a layer stays FMA, multiply, exp2, add, reciprocal, FMA,
// sign, select.
// bf16 activations: the hardware tanh approximation (relative error about 1e-5,
// far below bfloat16's 2^-9), since the result is rounded to bf16 right after.
constexpr float kTwoLog2e = 2.88539008177792681f;

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
  float y;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float tanh_approx(float x) {
  float y;
  asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
template <bool BF16>
__device__ __forceinline__ float round_to(float v) {
  if constexpr (BF16) return __bfloat162float(__float2bfloat16_rn(v));
  else return v;
}
constexpr float kTanhPolyMax = 0.55f;
constexpr float kTanhP0 = 1.0f, kTanhP1 = -0.3333331048488617f, kTanhP2 = 0.1333247870206833f,
                kTanhP3 = -0.05384441092610359f, kTanhP4 = 0.021046100184321404f,
                kTanhP5 = -0.0062440442852675915f;
template <bool BF16>
__device__ __forceinline__ float block_tanh(float y) {
  if constexpr (BF16) return tanh_approx(y);
  const float ay = fabsf(y);
  const float big = copysignf(fmaf(-2.0f, rcp_approx(1.0f + ex2_approx(ay * kTwoLog2e)), 1.0f), y);
  const float q = y * y;
  float p = fmaf(kTanhP5, q, kTanhP4);
  p = fmaf(p, q, kTanhP3);
  p = fmaf(p, q, kTanhP2);
  p = fmaf(p, q, kTanhP1);
  p = fmaf(p, q, kTanhP0);
  return ay < kTanhPolyMax ? y * p : big;
}

// Hardware barriers in shared memory (mbarrier): arrive has release semantics
// and the parity wait acquire semantics at CTA scope, so slots written before an
// arrive are seen by a thread whose wait on that phase succeeded.
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_test(uint64_t* bar, int parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_try(uint64_t* bar, int parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_u32(bar)), "r"(parity), "r"(kSuspendHintNs) : "memory");
  return ok != 0;
}
// Bounded wait for the phase of `parity` to complete. The chain (critical path)
// polls; the tile warps let the hardware suspend them between checks. Gives up
// after `limit` checks, records the failure in *err and returns false, so no
// warp can wait forever (each check lasts at most kSuspendHintNs).
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, int parity, int* err, bool poll, int limit) {
  for (int it = 0; it < limit; ++it)
    if (poll ? mbar_test(bar, parity) : mbar_try(bar, parity)) return true;
  atomicExch(err, 1);
  return false;
}

// Warp roles. Chain warps (one stream per lane) run the red cells, blocks and
// sampler position after position. The layers form NG groups of K; after group k
// of position r every lane of chain warp c arrives on act_ready[k][c]. Tile warps
// own row groups (layer l, chain warp c): the gray block of step r for layer l
// needs a^{l-1} below r and must not run before the chain has consumed the
// accumulator of (r-1, l), so it waits for act_ready[group(l)] of position r-1,
// computes, and arrives on tile_done[group(l)][c] (which completes when every
// layer of the group has arrived); the chain waits on tile_done before reading a
// group's accumulators. Each barrier thus advances at most one phase ahead of
// its waiters, parity waits are exact, and every wait is bounded.
template <bool BF16, bool REC>
__global__ void __launch_bounds__(kChunkMaxThreads) k_chunk(Dims g, ChunkArgs a, int G) {
  extern __shared__ float csm[];
  const ChunkShape cs = chunk_shape(g, a.chunk, G);
  const int CH = cs.CH, CHP = cs.CHP, TPS = cs.TPS, GdMax = cs.GdMax, CW = cs.CW;
  float* win = csm + cs.win;   // [(M+1)][G][CHP]   slot window of positions [c, c+CH)
  float* tp = csm + cs.tp;     // [M][GdMax][TPS]   taps h[0..CH)
  float* h0s = csm + cs.h0;    // [M][GdMax]        h[0]
  float* ep = csm + cs.ep;     // [CH][G]           sampler noise
  float* ys = csm + cs.ys;     // [CH][G]           y^M of each position, written out at the end
  uint64_t* act_ready = reinterpret_cast<uint64_t*>(csm + cs.flags);   // [NG][CW]
  uint64_t* tile_done = act_ready + cs.NG * CW;                          // [NG][CW]
  const int K = cs.K, NG = cs.NG;
  const int M = g.M;
  const int s0 = blockIdx.x * G;
  const int Gc = min(G, g.S - s0);
  const int d_lo = s0 / g.B;
  const int Gd = (s0 + Gc - 1) / g.B - d_lo + 1;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int r0 = a.p0 - a.c, r1 = a.p1 - a.c;

  // Prologue: every load is an asynchronous 4-byte copy into shared memory
  // (zero-filled where the slot holds nothing yet), so the loads of a thread
  // overlap instead of waiting one by one on HBM latency. Rows are spread over
  // warps and positions over lanes, so index arithmetic is per row.
  const int wid = tid >> 5, lid = tid & 31, nw = nt >> 5;
  for (int row = wid; row < M * Gd; row += nw) {
    const int l = row / Gd, dl = row - l * Gd;
    const float* src = a.taps + ((size_t)l * g.D + d_lo + dl) * g.L;
    float* dst = tp + (l * GdMax + dl) * TPS;
    for (int j = lid; j < CH; j += 32) cp_async4(dst + j, src + j, true);
  }
  // Slots already in HBM: tokens and activations below p0; the token at p0 when
  // no x0 is given; accumulators that some block has reached (the first block to
  // reach position t runs at step highbit(t)). Everything else starts at 0.
  for (int row = wid; row < (M + 1) * Gc; row += nw) {
    const int l = row / Gc, gg = row - l * Gc;
    const float* src = a.state + slot_index(g, l, s0 + gg, 0);
    float* dst = win + (l * G + gg) * CHP;
    for (int r = lid; r < CH; r += 32) {
      const int t = a.c + r;
      bool valid = false;
      if (t < g.L) {
        valid = t < a.p0;
        if (l == 0) valid = valid || (t == a.p0 && a.x0 == nullptr);
        else valid = valid || (t >= 1 && highbit_dev(t) <= a.last_done);
      }
      cp_async4(dst + r, src + (valid ? t : 0), valid);
    }
  }
  for (int r = r0 + wid; r < r1; r += nw) {
    const float* src = a.eps + (size_t)(a.c + r - a.gen_base) * g.S;
    for (int gg = lid; gg < Gc; gg += 32) {
      const int s = s0 + gg, d = s / g.B, b = s - d * g.B;
      cp_async4(ep + r * G + gg, src + (size_t)b * g.D + d, true);
    }
  }
  cp_async_wait_all();
  __syncthreads();
  for (int k = tid; k < M * Gd; k += nt) {
    const int dl = k % Gd, l = k / Gd;
    h0s[l * GdMax + dl] = tp[(l * GdMax + dl) * TPS];
  }
  if (a.x0 != nullptr && tid < Gc) {
    const int s = s0 + tid, d = s / g.B, b = s - d * g.B;
    win[tid * CHP + r0] = round_act(load_token(a.x0, (size_t)b * g.D + d, g.bf16), g.bf16);
  }
  for (int k = tid; k < NG * CW; k += nt) {
    const int grp = k / CW;
    mbar_init(act_ready + k, 32);
    mbar_init(tile_done + k, 32 * (min(M, (grp + 1) * K) - grp * K));   // one arrival per lane per layer
  }
  __syncthreads();

  const int warp = tid >> 5, lane = tid & 31;
  const int rs = r0 > 0 ? r0 : 1;   // first position of this launch with an on-chip gray block
  int* err = a.err;
  bool ok = true;
  if (warp < CW) {
    // ---------------------------------------------------------------- chain warp
    // Lanes past the CTA's last stream read stream 0's slots so that every load
    // is valid, and store nothing (stores are predicated on `act`).
    const int gg0 = warp * 32 + lane;
    const bool act = gg0 < Gc;
    const int gg = act ? gg0 : 0;
    const int s = s0 + gg, d = s / g.B, b = s - d * g.B;
    const int c_dl = d - d_lo;
    const size_t c_io = (size_t)b * g.D + d;
    const int lstride = G * CHP;                 // window floats per layer
    float* wrow = win + gg * CHP;                // this stream's row of layer 0
    const float* hrow = h0s + c_dl;              // h0 of layer l at (l-1)*GdMax
    float av = wrow[r0];                         // the token of the current position
    // Barrier tests run one group ahead (non-blocking), so their latency hides
    // behind the previous group's layers; a test that comes back false is
    // followed by a bounded wait.
    bool ready = r0 == 0;                        // group 0 of position r0 needs no wait when r0 == 0
    if (!ready) ready = mbar_test(&tile_done[warp], 0);
    for (int r = r0; r < r1; ++r) {
      const int t = a.c + r;
      const float epsv = ep[r * G + gg];
      float y = 0.f;
      for (int grp = 0; grp < NG; ++grp) {
        const int lg0 = grp * K + 1, lg1 = min(M, (grp + 1) * K);
        if (!ready && ok) ok = mbar_wait(&tile_done[grp * CW + warp], (r - rs) & 1, err, true, a.wait_limit);
        const int lend = lg1 < M ? lg1 : M - 1;    // layers with a block (tanh) in this group
        float acc = wrow[lg0 * lstride + r];
        float h0 = hrow[(lg0 - 1) * GdMax];
        auto layer = [&](int l) {
          const int ln = l < lg1 ? l + 1 : l;      // prefetch the next layer of the group
          const float acc_n = wrow[ln * lstride + r];
          const float h0_n = hrow[(ln - 1) * GdMax];
          y = fmaf(h0, av, acc);
          if constexpr (REC) if (act) a.rec[((size_t)(l - 1) * a.n_gen + (t - a.gen_base)) * g.S + c_io] = y;
          av = round_to<BF16>(block_tanh<BF16>(y));
          if (act) wrow[l * lstride + r] = av;
          acc = acc_n;
          h0 = h0_n;
        };
        // Halfway through the group, test the next group's barrier (the next
        // position's group 0 after the last group); by then its blocks are
        // usually done, and the test's latency hides behind the second half.
        const int lmid = lg0 + (lend - lg0 + 1) / 2;
        for (int l = lg0; l < lmid; ++l) layer(l);
        {
          const int ng = grp + 1 < NG ? grp + 1 : 0;
          const int nr = grp + 1 < NG ? r : r + 1;
          ready = (nr == 0 || nr >= r1) ? true : mbar_test(&tile_done[ng * CW + warp], (nr - rs) & 1);
        }
        for (int l = lmid; l <= lend; ++l) layer(l);
        if (lg1 == M) {                            // last layer: red cell only
          y = fmaf(h0, av, acc);
          if constexpr (REC) if (act) a.rec[((size_t)(M - 1) * a.n_gen + (t - a.gen_base)) * g.S + c_io] = y;
        }
        mbar_arrive(&act_ready[grp * CW + warp]);
      }
      if (act) ys[r * G + gg] = y;
      // x_{t+1}; for the last position of the chunk it lands in the row's spare
      // column (index CH) and goes to HBM with the write-back.
      av = round_to<BF16>(block_tanh<BF16>(y) + a.eps_scale * epsv);
      if (act && t + 1 < g.L) wrow[r + 1] = av;
    }
  } else {
    // ---------------------------------------------------------------- tile warps
    // With a single chain warp, tile work stays off the scheduler that issues
    // for it (warp w issues on scheduler w % 4), so the latency-bound chain
    // shares its issue slots with no busy warp; that leaves 12 of the 15 other
    // warps for blocks (measured on the headline shape: 7.6 % fewer cycles per
    // chunk). With more chain warps every warp takes blocks.
    const int nwarps = nt / 32;
    const bool spare_sched = CW == 1 && nwarps - CW > 4;
    auto is_tile = [&](int w) { return w >= CW && (!spare_sched || (w & 3) >= CW); };
    int tw = 0, ntw = 0;
    for (int w = CW; w < nwarps; ++w)
      if (is_tile(w)) {
        if (w < warp) ++tw;
        ++ntw;
      }
    if (is_tile(warp))
    for (int r = rs; r < r1; ++r) {
      const int U = r & -r;
      for (int k = tw; k < M * CW; k += ntw) {
        const int l = k / CW + 1, c = k - (l - 1) * CW;
        const int grp = (l - 1) / K;
        if (r > r0 && ok) ok = mbar_wait(&act_ready[grp * CW + c], (r - 1 - r0) & 1, err, false, a.wait_limit);
        const int gg = c * 32 + lane;
        if (gg < Gc) {
          const int dl = (s0 + gg) / g.B - d_lo;
          gray_block(U, win + ((l - 1) * G + gg) * CHP, win + (l * G + gg) * CHP, tp + ((l - 1) * GdMax + dl) * TPS, r);
        }
        mbar_arrive(&tile_done[grp * CW + c]);
      }
    }
  }
  __syncthreads();

  // Outputs of the positions produced, then the next chunk's first token.
  const int wid2 = tid >> 5, lid2 = tid & 31, nw2 = nt >> 5;
  for (int r = r0 + wid2; r < r1; r += nw2) {
    float* dst = a.y_out + (size_t)(a.c + r - a.gen_base) * g.S;
    for (int gg = lid2; gg < Gc; gg += 32) {
      const int s = s0 + gg, d = s / g.B, b = s - d * g.B;
      dst[(size_t)b * g.D + d] = ys[r * G + gg];
    }
  }
  if (r1 == CH && a.c + CH < g.L && tid < Gc) a.state[slot_index(g, 0, s0 + tid, a.c + CH)] = win[tid * CHP + CH];
  // Write back positions [p0, c+CH) of layers 0..M-1: new tokens and
  // activations below p1, accumulators (including the small blocks' partial
  // sums) from p1 on. Layer M's slots below p1 were consumed and nothing reads
  // them again; its accumulators from p1 on are still needed.
  for (int row = wid2; row < (M + 1) * Gc; row += nw2) {
    const int l = row / Gc, gg = row - l * Gc;
    float* dst = a.state + slot_index(g, l, s0 + gg, a.c);
    const float* src = win + (l * G + gg) * CHP;
    const int rb = l == M ? r1 : r0;            // first slot to write
    const int re = min(CH, g.L - a.c);          // past the last
    if ((a.c & 3) == 0 && (rb & 3) == 0 && (re & 3) == 0) {
      for (int q = (rb >> 2) + lid2; q < (re >> 2); q += 32) {
        const int r = 4 * q;
        reinterpret_cast<float4*>(dst)[q] = make_float4(src[r], src[r + 1], src[r + 2], src[r + 3]);
      }
    } else {
      for (int r = rb + lid2; r < re; r += 32) dst[r] = src[r];
    }
  }
}

size_t chunk_smem_bytes(const Dims& g, int chunk, int G) { return chunk_shape(g, chunk, G).total * sizeof(float); }

static int chunk_threads(const Dims& g, int G) {
  const int cw = (G + 31) / 32;
  int tile_warps = g.M * cw;
  if (tile_warps > kChunkMaxThreads / 32 - cw) tile_warps = kChunkMaxThreads / 32 - cw;
  return 32 * (cw + tile_warps);
}

int chunk_streams_per_cta(const Dims& g, int chunk, int num_sms, size_t max_smem) {
  int G = (g.S + num_sms - 1) / num_sms;
  if (G > kChunkMaxStreams) G = kChunkMaxStreams;
  if (G < 1) G = 1;
  auto fits = [&](int G_) {
    const int cw = (G_ + 31) / 32;
    return chunk_smem_bytes(g, chunk, G_) <= max_smem && kChunkMaxThreads / 32 - cw >= 1;
  };
  while (G > 1 && !fits(G)) G = (G + 1) / 2;
  if (!fits(G)) return 0;
  return G;
}

// The dynamic shared-memory cap is one value per kernel function and device,
// shared by every context in the process; it only ever grows here, so a small
// configuration never lowers it under a live context that needs more.
template <class K>
static cudaError_t raise_smem_cap(K kernel, size_t smem) {
  cudaFuncAttributes fa{};
  cudaError_t e = cudaFuncGetAttributes(&fa, kernel);
  if (e != cudaSuccess) return e;
  if ((size_t)fa.maxDynamicSharedSizeBytes >= smem) return cudaSuccess;
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
}

cudaError_t configure_chunk(size_t smem) {
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  cudaError_t e = raise_smem_cap(k_chunk<false, false>, smem);
  if (e == cudaSuccess) e = raise_smem_cap(k_chunk<false, true>, smem);
  if (e == cudaSuccess) e = raise_smem_cap(k_chunk<true, false>, smem);
  if (e == cudaSuccess) e = raise_smem_cap(k_chunk<true, true>, smem);
  return e;
}

cudaError_t launch_chunk(const Dims& g, const ChunkArgs& a, int G, cudaStream_t st) {
  const size_t smem = chunk_smem_bytes(g, a.chunk, G);
  const int blocks = (g.S + G - 1) / G;
  const int nt = chunk_threads(g, G);
  if (g.bf16) {
    if (a.rec) k_chunk<true, true><<<blocks, nt, smem, st>>>(g, a, G);
    else k_chunk<true, false><<<blocks, nt, smem, st>>>(g, a, G);
  } else {
    if (a.rec) k_chunk<false, true><<<blocks, nt, smem, st>>>(g, a, G);
    else k_chunk<false, false><<<blocks, nt, smem, st>>>(g, a, G);
  }
  return cudaGetLastError();
}

}  // namespace fi
