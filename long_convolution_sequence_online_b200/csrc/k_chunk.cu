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
// Re-timed on-chip blocks. Inside the chunk every block is a direct sum, whose
// cost is its area whatever the tiling, so the blocks of side >= 16 (the 16 x 16
// and 32 x 32 blocks of the page's tiling, which would otherwise stall the
// chain for thousands of cycles at their step) are cut into pieces that run
// when their inputs exist and before their outputs are read: for the block of
// step r and side U, with H = U/2,
//   sources [r-U, r-H) -> targets [r, r+U)     run at steps r-H+1, r-H+3, ... < r,
//   sources [r-H, r)   -> targets [r+H, r+U)   run at steps r+1, r+3, ...  < r+H,
//   sources [r-H, r)   -> targets [r, r+H)     the same cut again, down to 8 x 8 at step r.
// Every (source, target) pair of the chunk is still summed exactly once (the
// host builds the table; tests/test_abi.py checks it). A launch that covers only
// part of a chunk (a call boundary inside it) keeps the page's tiling unchanged,
// so the state between calls is the same whichever call sequence produced it.
//
// Shared-memory window: position-major per layer, win[l][r][gg] (gg = stream in
// the CTA), so the chain (one stream per lane) and the tile warps (one stream
// per lane, sliding over positions) both touch 32 consecutive floats per warp
// access, and the prologue and write-back move 16 contiguous bytes of a stream
// per lane.
#include <algorithm>
#include <mutex>
#include <vector>

#include "fi_internal.cuh"

namespace fi {

constexpr int kChunkMaxThreads = 512;
constexpr int kChunkMaxStreams = 128;
constexpr int kSuspendHintNs = 1000;   // longest a suspended barrier check may last
constexpr int kRing = 4;                // depth of the hand-off barrier rings
static_assert(kChainLags >= 1 && kChainLags <= 3, "the chain holds h[0..3] in one 16-byte load");
static_assert(kRing >= kChainLags + 1, "a ring slot must never get two phases ahead of its waiter");

struct ChunkShape {
  int G, GP, CH, LS, TPS, CW, GdMax, NG, K;
  size_t win, tp, hv, ep, flags, total;  // float offsets / total floats
};

__host__ __device__ inline ChunkShape chunk_shape(const Dims& g, int CH, int G) {
  ChunkShape c;
  c.G = G;
  c.GP = G | 1;                    // odd: the prologue's transposing stores spread over banks
  c.CH = CH;
  // floats per layer: the chunk's positions plus kChainLags spare ones (the next
  // chunk's token, and targets of pieces that reach past the chunk)
  c.LS = (CH + kChainLags) * c.GP;
  c.TPS = (CH + kChainLags) | 1;   // odd tap stride: lanes of different channels hit different banks
  c.CW = (G + 31) / 32;            // chain warps (one stream per lane)
  c.GdMax = (G - 1) / g.B + 2;     // channels a run of G consecutive streams can touch
  c.NG = 1;                        // one hand-off per position (both ways)
  c.K = g.M;
  c.win = 0;
  c.tp = c.win + (size_t)(g.M + 1) * c.LS;
  c.hv = (c.tp + (size_t)g.M * c.GdMax * c.TPS + 3) & ~(size_t)3;   // 16-byte aligned
  c.ep = c.hv + (size_t)4 * g.M * c.GdMax;
  c.flags = (c.ep + (size_t)CH * G + 1) & ~(size_t)1;   // 8-byte aligned mbarriers
  c.total = c.flags + 2 * (size_t)(2 * kRing) * c.CW;  // act_ready[kRing][CW] + tile_done[kRing][CW]
  return c;
}

__device__ __forceinline__ int highbit_dev(int t) { return 1 << (31 - __clz(t)); }

// 4-byte asynchronous global -> shared copy.
__device__ __forceinline__ void cp_async4(float* dst, const float* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// ---------------------------------------------------------------------------
// Step table: which on-chip block pieces run at which step (host-built).
// ---------------------------------------------------------------------------
enum PieceKind { PK_SQ1 = 0, PK_SQ2, PK_SQ4, PK_SQ8, PK_SQ16, PK_SQ32, PK_R8x4, PK_R16x4, PK_R16x2, PK_COUNT };
__host__ __device__ constexpr int piece_ns(int k) {
  return k == PK_R8x4 ? 8 : (k == PK_R16x4 || k == PK_R16x2) ? 16 : 1 << k;
}
__host__ __device__ constexpr int piece_nd(int k) { return k == PK_R16x2 ? 2 : k >= PK_R8x4 ? 4 : 1 << k; }
__host__ __device__ inline uint32_t piece_encode(int step, int s_lo, int t_lo, int kind) {
  return (uint32_t)step | ((uint32_t)s_lo << 7) | ((uint32_t)t_lo << 14) | ((uint32_t)kind << 21);
}

// Block piece: dst[t] += sum_{s in [s_lo, s_lo+NS)} h[t-s] src[s] for t in
// [t_lo, t_lo+ND), positions `stride` floats apart. Outputs go in groups of OB;
// within a group the taps h[t-s] form a window that slides by one per source, so
// each source costs one source load, one tap load and OB FMAs from registers.
template <int NS, int ND>
__device__ __forceinline__ void block_piece(const float* __restrict__ src, float* __restrict__ dst,
                                            const float* __restrict__ taps, int s_lo, int t_lo, int stride) {
  constexpr int OB = ND < 8 ? ND : 8;
  const float* x = src + s_lo * stride;
#pragma unroll
  for (int o0 = 0; o0 < ND; o0 += OB) {
    const int lag0 = t_lo + o0 - s_lo;     // lag of output o0 + k for source 0 is lag0 + k
    float acc[OB], w[OB];
#pragma unroll
    for (int k = 0; k < OB; ++k) {
      acc[k] = 0.f;
      w[k] = taps[lag0 + k];
    }
#pragma unroll
    for (int u = 0; u < NS; ++u) {
      const float xv = x[u * stride];
#pragma unroll
      for (int k = 0; k < OB; ++k) acc[k] = fmaf(w[k], xv, acc[k]);
      if (u + 1 < NS) {
#pragma unroll
        for (int k = OB - 1; k > 0; --k) w[k] = w[k - 1];
        w[0] = taps[lag0 - u - 1];
      }
    }
    float* out = dst + (t_lo + o0) * stride;
#pragma unroll
    for (int k = 0; k < OB; ++k) out[k * stride] += acc[k];
  }
}

__device__ __forceinline__ void run_piece(uint32_t e, const float* src, float* dst, const float* taps, int stride);

// The same piece for two rows (two layers of one stream) at once: two
// independent FMA chains per output group, so a warp with two rows pays the
// latency of one.
template <int NS, int ND>
__device__ __forceinline__ void block_piece2(const float* __restrict__ srcA, float* __restrict__ dstA,
                                             const float* __restrict__ tapsA, const float* __restrict__ srcB,
                                             float* __restrict__ dstB, const float* __restrict__ tapsB, int s_lo,
                                             int t_lo, int stride) {
  constexpr int OB = ND < 8 ? ND : 8;
  const float* xA = srcA + s_lo * stride;
  const float* xB = srcB + s_lo * stride;
#pragma unroll
  for (int o0 = 0; o0 < ND; o0 += OB) {
    const int lag0 = t_lo + o0 - s_lo;
    float accA[OB], wA[OB], accB[OB], wB[OB];
#pragma unroll
    for (int k = 0; k < OB; ++k) {
      accA[k] = 0.f;
      accB[k] = 0.f;
      wA[k] = tapsA[lag0 + k];
      wB[k] = tapsB[lag0 + k];
    }
#pragma unroll
    for (int u = 0; u < NS; ++u) {
      const float xa = xA[u * stride], xb = xB[u * stride];
#pragma unroll
      for (int k = 0; k < OB; ++k) {
        accA[k] = fmaf(wA[k], xa, accA[k]);
        accB[k] = fmaf(wB[k], xb, accB[k]);
      }
      if (u + 1 < NS) {
#pragma unroll
        for (int k = OB - 1; k > 0; --k) {
          wA[k] = wA[k - 1];
          wB[k] = wB[k - 1];
        }
        wA[0] = tapsA[lag0 - u - 1];
        wB[0] = tapsB[lag0 - u - 1];
      }
    }
    float* outA = dstA + (t_lo + o0) * stride;
    float* outB = dstB + (t_lo + o0) * stride;
#pragma unroll
    for (int k = 0; k < OB; ++k) {
      outA[k * stride] += accA[k];
      outB[k * stride] += accB[k];
    }
  }
}

// Dispatch by kind with direct branches, the kinds of the whole-chunk tables
// first (measured ~2 % faster per launch than a switch's indirect jump).
__device__ __forceinline__ void run_piece2(uint32_t e, const float* srcA, float* dstA, const float* tapsA,
                                           const float* srcB, float* dstB, const float* tapsB, int stride) {
  const int s_lo = (e >> 7) & 127, t_lo = (e >> 14) & 127;
  const int k = (e >> 21) & 15;
  if (k == PK_SQ1) block_piece2<1, 1>(srcA, dstA, tapsA, srcB, dstB, tapsB, s_lo, t_lo, stride);
  else if (k == PK_SQ8) block_piece2<8, 8>(srcA, dstA, tapsA, srcB, dstB, tapsB, s_lo, t_lo, stride);
  else if (k == PK_SQ2) block_piece2<2, 2>(srcA, dstA, tapsA, srcB, dstB, tapsB, s_lo, t_lo, stride);
  else if (k == PK_R16x4) block_piece2<16, 4>(srcA, dstA, tapsA, srcB, dstB, tapsB, s_lo, t_lo, stride);
  else if (k == PK_SQ4) block_piece2<4, 4>(srcA, dstA, tapsA, srcB, dstB, tapsB, s_lo, t_lo, stride);
  else {
    run_piece(e, srcA, dstA, tapsA, stride);
    run_piece(e, srcB, dstB, tapsB, stride);
  }
}

__device__ __forceinline__ void run_piece(uint32_t e, const float* src, float* dst, const float* taps, int stride) {
  const int s_lo = (e >> 7) & 127, t_lo = (e >> 14) & 127;
  const int k = (e >> 21) & 15;
  if (k == PK_SQ1) block_piece<1, 1>(src, dst, taps, s_lo, t_lo, stride);
  else if (k == PK_SQ8) block_piece<8, 8>(src, dst, taps, s_lo, t_lo, stride);
  else if (k == PK_SQ2) block_piece<2, 2>(src, dst, taps, s_lo, t_lo, stride);
  else if (k == PK_R16x4) block_piece<16, 4>(src, dst, taps, s_lo, t_lo, stride);
  else if (k == PK_SQ4) block_piece<4, 4>(src, dst, taps, s_lo, t_lo, stride);
  else if (k == PK_SQ16) block_piece<16, 16>(src, dst, taps, s_lo, t_lo, stride);
  else if (k == PK_SQ32) block_piece<32, 32>(src, dst, taps, s_lo, t_lo, stride);
  else if (k == PK_R8x4) block_piece<8, 4>(src, dst, taps, s_lo, t_lo, stride);
  else block_piece<16, 2>(src, dst, taps, s_lo, t_lo, stride);
}

namespace {

int kind_of_square(int U) { return U == 1 ? PK_SQ1 : U == 2 ? PK_SQ2 : U == 4 ? PK_SQ4 : U == 8 ? PK_SQ8 : U == 16 ? PK_SQ16 : PK_SQ32; }

struct Piece { int step, s_lo, t_lo, kind; };

// The block of step r and side U (sources [r-U, r), targets from r + sh), cut
// so that at most an 8 x 8 square is bound to step r itself (see the file
// comment): with H = U/2, sources [r-U, r-H) to every target, sources [r-H, r)
// to the targets past r+H+sh, and the square [r-H, r) x [r+sh, r+H+sh) cut
// again. The other pieces get a step later (balance_pieces). Blocks of side 8
// stay whole: each piece costs a fixed ~200 cycles on top of its products
// (measured with clock stamps on B200), so one 64-product piece beats four of 16.
void cut_block(int r, int U, int sh, bool coarse, std::vector<Piece>& out) {
  if (U <= 8) {
    out.push_back({r, r - U, r + sh, kind_of_square(U)});
    return;
  }
  const int H = U / 2;
  // 64 products per row (measured on B200: pieces of 32 products took more
  // steps' worth of per-piece latency than they saved); with a short chain
  // (few layers) the tile warps set the pace and 16 x 16 pieces measured faster
  const int kind = H == 16 ? (coarse ? PK_SQ16 : PK_R16x4) : H == 8 ? PK_SQ8 : PK_SQ4;
  const int nd = piece_nd(kind);
  for (int t = r + sh; t < r + sh + U; t += nd) out.push_back({-1, r - U, t, kind});
  for (int t = r + H + sh; t < r + U + sh; t += nd) out.push_back({-1, r - H, t, kind});
  cut_block(r, H, sh, coarse, out);
}

// A piece reading sources [s_lo, s_lo+ns) and writing targets from t_lo may run
// at any step k with s_lo + ns <= k <= t_lo - sh. Pieces with a step already
// fixed keep it; each other piece, the tightest windows first, goes to the
// least loaded step of its window (load = products per row plus a fixed cost
// per piece), so every step carries about the same work.
void balance_pieces(std::vector<Piece>& p, int CH, int sh) {
  constexpr int kPieceCost = 8;
  std::vector<int> load(CH + kChainLags, 0);
  for (const Piece& x : p)
    if (x.step >= 0) load[x.step] += piece_ns(x.kind) * piece_nd(x.kind) + kPieceCost;
  std::vector<Piece*> free_p;
  for (Piece& x : p)
    if (x.step < 0) free_p.push_back(&x);
  auto lo = [](const Piece* x) { return x->s_lo + piece_ns(x->kind); };
  auto hi = [&](const Piece* x) { return x->t_lo - sh; };
  std::stable_sort(free_p.begin(), free_p.end(), [&](const Piece* a, const Piece* b) {
    const int wa = hi(a) - lo(a), wb = hi(b) - lo(b);
    return wa != wb ? wa < wb : lo(a) < lo(b);
  });
  for (Piece* x : free_p) {
    int best = lo(x);
    for (int k = lo(x); k <= hi(x) && k < CH; ++k)
      if (load[k] < load[best]) best = k;
    x->step = best;
    load[best] += piece_ns(x->kind) * piece_nd(x->kind) + kPieceCost;
  }
}

}  // namespace

int chunk_piece_sources(int kind) { return piece_ns(kind); }
int chunk_piece_targets(int kind) { return piece_nd(kind); }

bool build_chunk_table(int CH, bool retimed, ChunkTable* tab, bool coarse) {
  std::vector<Piece> p;
  const int sh = retimed ? kChainLags : 0;   // retimed: the chain takes lags 1..sh, pieces the rest
  for (int r = 1; r < CH; ++r) {
    const int U = r & -r;
    std::vector<Piece> q;
    if (retimed) cut_block(r, U, sh, coarse, q);
    else q.push_back({r, r - U, r, kind_of_square(U)});
    // pieces whose targets all lie past the chunk are dropped; one that reaches
    // past it writes its last targets into the window's spare positions (CH and
    // up), which nothing reads
    for (const Piece& x : q)
      if (x.t_lo < CH) p.push_back(x);
  }
  if (retimed) balance_pieces(p, CH, sh);
  if ((int)p.size() > kChunkMaxEntries) return false;
  std::stable_sort(p.begin(), p.end(), [](const Piece& a, const Piece& b) { return a.step < b.step; });
  tab->n = (int)p.size();
  tab->lag1 = sh;
  int k = 0;
  for (int r = 0; r <= kChunkMaxSteps; ++r) {
    while (k < tab->n && p[k].step < r) ++k;
    tab->first[r] = (uint16_t)k;
  }
  for (int j = 0; j < tab->n; ++j) tab->e[j] = piece_encode(p[j].step, p[j].s_lo, p[j].t_lo, p[j].kind);
  return true;
}

// ---------------------------------------------------------------------------
// tanh for the block and the sampler, without branches (every lane of the chain
// warp takes the same path).
// fp32 activations: two forms evaluated side by side and selected by |y|.
//  * |y| >= 0.55: tanh y = 1 - 2 rc, rc = 1 / (1 + e^(2y)), with the hardware
//    exp2 and reciprocal, e^(2y) = 2^(2y log2 e). For y >= 0.55, 2 rc <= 0.5 and
//    the subtraction loses nothing; for y <= -0.55, |tanh y| >= 0.5 and the
//    rounding of 2 rc is at most an ulp of 2. Overflow of e^(2y) to +inf gives
//    rc = 0 (tanh = 1), underflow to 0 gives rc = 1 (tanh = -1).
//  * |y| < 0.55: y * P(y^2), P a degree-5 polynomial fitted to tanh(y)/y by
//    weighted least squares on that interval (fit error 1e-9).
// Relative error within about 5e-7 for every y (1e-7 in the polynomial range).
// The chain never forms tanh(y) on its critical path: the next layer's input
// y' = h0' tanh(y) + acc' is taken straight from the parts, as
// y' = (h0' + acc') - 2 h0' rc, or h0' (y P) + acc', so each layer costs the
// exp2 / add / reciprocal / FMA / select chain (the polynomial runs beside it);
// the argument of the next exp2 (2 log2 e y') comes out of the same FMAs.
// bf16 activations: the hardware tanh approximation (relative error about 1e-5,
// far below bfloat16's 2^-9), since the result is rounded to bf16 right after.
// ---------------------------------------------------------------------------
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
__device__ __forceinline__ float round_bf16(float v) { return __bfloat162float(__float2bfloat16_rn(v)); }

constexpr float kTanhPolyMax = 0.55f;
constexpr float kTanhP0 = 1.0f, kTanhP1 = -0.3333331048488617f, kTanhP2 = 0.1333247870206833f,
                kTanhP3 = -0.05384441092610359f, kTanhP4 = 0.021046100184321404f,
                kTanhP5 = -0.0062440442852675915f;

// tanh(y) in parts, from y and z = 2 log2(e) y.
struct TanhParts {
  float rc;    // 1 / (1 + e^(2y))
  float tp;    // y P(y^2)
  bool small;  // |y| < kTanhPolyMax: tanh y = tp, else 1 - 2 rc
};
__device__ __forceinline__ TanhParts tanh_parts(float y, float z) {
  TanhParts p;
  p.rc = rcp_approx(1.0f + ex2_approx(z));
  const float q = y * y;
  float pp = fmaf(kTanhP5, q, kTanhP4);
  pp = fmaf(pp, q, kTanhP3);
  pp = fmaf(pp, q, kTanhP2);
  pp = fmaf(pp, q, kTanhP1);
  pp = fmaf(pp, q, kTanhP0);
  p.tp = y * pp;
  p.small = fabsf(y) < kTanhPolyMax;
  return p;
}
__device__ __forceinline__ float tanh_value(const TanhParts& p) { return p.small ? p.tp : fmaf(-2.0f, p.rc, 1.0f); }
// y' = h0 tanh(y) + acc and z' = 2 log2(e) y', from the parts of tanh(y).
__device__ __forceinline__ void next_input(const TanhParts& p, float h0, float acc, float& y, float& z) {
  const float c1 = h0 + acc;
  const float m2 = -2.0f * h0;
  const float yb = fmaf(m2, p.rc, c1);
  const float zb = fmaf(kTwoLog2e * m2, p.rc, kTwoLog2e * c1);
  const float yp = fmaf(h0, p.tp, acc);
  const float zp = fmaf(kTwoLog2e * h0, p.tp, kTwoLog2e * acc);
  y = p.small ? yp : yb;
  z = p.small ? zp : zb;
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
  if (mbar_test(bar, parity)) return true;   // already complete: no suspend round trip
  for (int it = 0; it < limit; ++it)
    if (poll ? mbar_test(bar, parity) : mbar_try(bar, parity)) return true;
  atomicExch(err, 1);
  return false;
}

// Warp roles. Chain warps (one stream per lane) run the red cells, blocks and
// sampler position after position. The layers form NG groups of K; after group k
// of position r every lane of chain warp c arrives on act_ready[k][c]. Tile warps
// own row groups (layer l, chain warp c): the pieces of step r for layer l need
// a^{l-1} below r and must not run before the chain has consumed the
// accumulator of (r-1, l), so they wait for act_ready[group(l)] of position r-1,
// compute, and arrive on tile_done[group(l)][c] (which completes when every
// layer of the group has arrived); the chain waits on tile_done before reading a
// group's accumulators. Each barrier thus advances at most one phase ahead of
// its waiters, parity waits are exact, and every wait is bounded.
// TRIG: the variant that lets the next block launch (programmatic) start once
// every CTA holds its window; launches followed by a plain block launch use the
// variant without the instruction.
template <bool BF16, bool REC, bool TRIG>
__global__ void __launch_bounds__(kChunkMaxThreads) k_chunk(Dims g, ChunkArgs a, int G) {
  extern __shared__ float csm[];
  const ChunkShape cs = chunk_shape(g, a.chunk, G);
  const int CH = cs.CH, GP = cs.GP, LS = cs.LS, TPS = cs.TPS, GdMax = cs.GdMax, CW = cs.CW;
  float* win = csm + cs.win;   // [(M+1)][CH+1][GP]   slot window of positions [c, c+CH]
  float* tp = csm + cs.tp;     // [M][GdMax][TPS]     taps h[0..CH), zero above
  float* ep = csm + cs.ep;     // [CH][G]             sampler noise
  float4* hv4 = reinterpret_cast<float4*>(csm + cs.hv);   // [M][GdMax] (h[0], h[1], h[2], h[3]) for the chain
  // Hand-off barrier rings (ordinal o uses slot o % kRing, phase parity
  // (o / kRing) & 1): act_ready[k][c] completes when chain warp c has finished a
  // position, tile_done[k][c] when every layer's pieces of a step are done for
  // chain warp c's streams. The chain runs at most kChainLags + 1 positions
  // ahead of the tile warps and they at most one step ahead of it, so a ring
  // slot never gets two phases ahead of its waiters.
  uint64_t* act_ready = reinterpret_cast<uint64_t*>(csm + cs.flags);   // [kRing][CW]
  uint64_t* tile_done = act_ready + kRing * CW;                          // [kRing][CW]
  const int M = g.M;
  const int s0 = blockIdx.x * G;
  const int Gc = min(G, g.S - s0);
  const int d_lo = s0 / g.B;
  const int Gd = (s0 + Gc - 1) / g.B - d_lo + 1;
  const int tid = threadIdx.x, nt = blockDim.x;
  const int r0 = a.p0 - a.c, r1 = a.p1 - a.c;

  // ---------------------------------------------------------------- prologue
  // Slots already in HBM: tokens and activations below p0; the token at p0 when
  // no x0 is given; accumulators that some block has reached (the first block to
  // reach position t runs at step highbit(t)). Everything else starts at 0.
  // Each lane moves 16 contiguous bytes (4 positions of one stream) and spreads
  // them over the position-major window; loads are issued in batches of 8 so a
  // thread has several in flight.
  auto slot_valid = [&](int l, int t) {
    if (t < a.p0) return true;
    if (l == 0) return t == a.p0 && a.x0 == nullptr;
    return t >= 1 && highbit_dev(t) <= a.last_done;
  };
  {
    const int wid = tid >> 5, lid = tid & 31, nw = nt >> 5;
    for (int r = r0 + wid; r < r1; r += nw) {
      const float* src = a.eps + (size_t)(a.c + r - a.gen_base) * g.S;
      for (int gg = lid; gg < Gc; gg += 32) {
        const int s = s0 + gg, d = s / g.B, b = s - d * g.B;
        cp_async4(ep + r * G + gg, src + (size_t)b * g.D + d);
      }
    }
  }
  // tp[.][CH]: the tap one past the window, zero (pieces that reach the spare
  // position read it)
  for (int k = tid; k < M * GdMax * (TPS - CH); k += nt) tp[(k / (TPS - CH)) * TPS + CH + k % (TPS - CH)] = 0.f;
  for (int k = tid; k < M * Gd; k += nt) {
    const int l = k / Gd, dl = k - l * Gd;
    const float* hrow = a.taps + ((size_t)l * g.D + d_lo + dl) * g.L;
    hv4[l * GdMax + dl] = g.L >= 4 ? __ldg(reinterpret_cast<const float4*>(hrow))
                                   : make_float4(hrow[0], g.L > 1 ? hrow[1] : 0.f, 0.f, 0.f);
  }
  // The taps and the noise are inputs no block writes, so they are fetched
  // before pdl_wait_primary() (while the preceding block launch drains); the
  // window, which that block writes, after it.
  if (CH < 4) {
    for (int idx = tid; idx < M * Gd * CH; idx += nt) {
      const int row = idx / CH, j = idx - row * CH;
      const int l = row / Gd, dl = row - l * Gd;
      tp[(l * GdMax + dl) * TPS + j] = a.taps[((size_t)l * g.D + d_lo + dl) * g.L + j];
    }
    pdl_wait_primary();
    for (int idx = tid; idx < (M + 1) * Gc * CH; idx += nt) {
      const int row = idx / CH, r = idx - row * CH;
      const int l = row / Gc, gg = row - l * Gc;
      const int t = a.c + r;
      win[l * LS + r * GP + gg] = slot_valid(l, t) ? a.state[slot_index(g, l, s0 + gg, t)] : 0.f;
    }
  } else {
    // Items: float4 j (4 positions or taps) of row `row` (a stream, or a
    // channel for the taps) of a layer, numbered with the rows padded to a
    // power of two, so a thread finds its item with shifts alone. Each thread
    // issues kBatch loads before storing any.
    const int vpr = CH >> 2;                          // float4 per row
    const int lv = 31 - __clz(vpr);
    const int lw = lv + (Gc > 1 ? 32 - __clz(Gc - 1) : 0);   // log2 items per window layer
    const int lt = lv + (Gd > 1 ? 32 - __clz(Gd - 1) : 0);   // log2 items per tap layer
    const int nwin = (M + 1) << lw, nall = nwin + (M << lt);
    constexpr int kBatch = 12;
    // items [nwin, nall) (taps) first, then [0, nwin) (window) after the wait
    for (int pass = 0; pass < 2; ++pass) {
      const int beg = pass == 0 ? nwin : 0, end = pass == 0 ? nall : nwin;
      if (pass == 1) pdl_wait_primary();
      for (int base = beg + tid; base < end; base += nt * kBatch) {
        float4 v[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int idx = base + u * nt;
          const bool is_win = idx < nwin;
          const int k = is_win ? idx : idx - nwin;
          const int sh = is_win ? lw : lt;
          const int l = k >> sh, rem = k & ((1 << sh) - 1);
          const int row = rem >> lv, j = rem & (vpr - 1);
          // every slot of the window lies inside the state, so the load is in
          // bounds; slots that hold nothing yet are zeroed below
          if (idx < end && row < (is_win ? Gc : Gd))
            v[u] = __ldg(reinterpret_cast<const float4*>(
                is_win ? a.state + slot_index(g, l, s0 + row, a.c + 4 * j)
                       : a.taps + ((size_t)l * g.D + d_lo + row) * g.L + 4 * j));
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int idx = base + u * nt;
          const bool is_win = idx < nwin;
          const int k = is_win ? idx : idx - nwin;
          const int sh = is_win ? lw : lt;
          const int l = k >> sh, rem = k & ((1 << sh) - 1);
          const int row = rem >> lv, j = rem & (vpr - 1);
          if (idx >= end || row >= (is_win ? Gc : Gd)) continue;
          if (is_win) {
            const int t = a.c + 4 * j;
            float* w = win + l * LS + 4 * j * GP + row;
            w[0] = slot_valid(l, t) ? v[u].x : 0.f;
            w[GP] = slot_valid(l, t + 1) ? v[u].y : 0.f;
            w[2 * GP] = slot_valid(l, t + 2) ? v[u].z : 0.f;
            w[3 * GP] = slot_valid(l, t + 3) ? v[u].w : 0.f;
          } else {
            float* w = tp + (l * GdMax + row) * TPS + 4 * j;
            w[0] = v[u].x;
            w[1] = v[u].y;
            w[2] = v[u].z;
            w[3] = v[u].w;
          }
        }
      }
    }
  }
  if (a.x0 != nullptr && tid < Gc) {
    const int s = s0 + tid, d = s / g.B, b = s - d * g.B;
    win[r0 * GP + tid] = round_act(load_token(a.x0, (size_t)b * g.D + d, g.bf16), g.bf16);
  }
  for (int k = tid; k < kRing * CW; k += nt) {
    mbar_init(act_ready + k, 32);
    mbar_init(tile_done + k, 32 * M);   // one arrival per lane per layer
  }
  cp_async_wait_all();
  __syncthreads();

  // Every CTA has its window: the next launch (the block at the next chunk
  // boundary, when launched programmatically) may start now; it waits for
  // this grid before reading.
  if constexpr (TRIG) pdl_launch_dependents();
  const int warp = tid >> 5, lane = tid & 31;
  // Hand-off. In the re-timed table the chain adds the terms of lags
  // 1..nlag (h^l[k] a^{l-1}_{t-k}) itself and the pieces of step i (sources
  // below i, targets from i+nlag) run while the chain is at positions i..,
  // needed at position i+nlag: the tile warps have nlag positions of slack.
  // Otherwise (a launch over part of a chunk, nlag = 0) the pieces of step i
  // have targets from i and the chain at position i waits for them.
  const int nlag = a.tab.lag1;
  const int rs = r0 > 0 ? r0 : 1;                 // first tile step
  const int s_last = nlag ? CH - 1 - nlag : r1 - 1;   // last tile step
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
    const size_t c_io = (size_t)b * g.D + d;
    const size_t y_stride = g.S;
    float* wcol = win + gg;                          // slot (l, r) at wcol[l*LS + r*GP]
    const float4* hv = hv4 + (d - d_lo);             // (h^l[0], h^l[1], h^l[2], .) at hv[(l-1)*HV]
    const int HV = GdMax;
    float x_cur = wcol[r0 * GP];                     // token of the current position (first: as loaded)
    TanhParts P{0.f, 0.f, true};
    float epsk = 0.f;                                // eps_scale * eps of the previous position
    bool from_parts = false;                         // layer 1's input is P (+ epsk), else x_cur
    for (int r = r0; r < r1; ++r) {
      const int t = a.c + r;
      // the pieces this position needs: step r - nlag
      const int need = r - nlag;
      if (need >= rs && need <= s_last && ok) {
        const int j = need - rs;
        ok = mbar_wait(&tile_done[(j % kRing) * CW + warp], (j / kRing) & 1, err, true, a.wait_limit);
      }
      // Lag terms the chain adds here: lag k only when its source lies in this
      // chunk (r >= k; earlier sources came with the blocks from HBM), applied
      // through 0/1 multipliers so the layer loop has no branch. The operands of
      // layer m (h^m[0..2] as one 16-byte load, the accumulator, a^{m-1} at
      // r-1 and r-2) are loaded two layers ahead of use, so their latency hides
      // behind two exp2/reciprocal chains.
      const float m1 = (nlag >= 1 && r >= 1) ? 1.f : 0.f;
      const float m2 = (nlag >= 2 && r >= 2) ? 1.f : 0.f;
      const float m3 = (nlag >= 3 && r >= 3) ? 1.f : 0.f;
      const int o1 = max(r - 1, 0) * GP, o2 = max(r - 2, 0) * GP, o3 = max(r - 3, 0) * GP, o0 = r * GP;
      float4 Hc = hv[0];
      float accc = wcol[LS + o0], a1c = wcol[o1], a2c = wcol[o2], a3c = kChainLags >= 3 ? wcol[o3] : 0.f;
      const int m_n = M >= 2 ? 2 : 1;
      float4 Hn = hv[(m_n - 1) * HV];
      float accn = wcol[m_n * LS + o0], a1n = wcol[(m_n - 1) * LS + o1], a2n = wcol[(m_n - 1) * LS + o2];
      float a3n = kChainLags >= 3 ? wcol[(m_n - 1) * LS + o3] : 0.f;
      auto acc_eff = [&](const float4& H, float acc, float a1, float a2, float a3) {
        float v = fmaf(m2 * H.z, a2, fmaf(m1 * H.y, a1, acc));
        if constexpr (kChainLags >= 3) v = fmaf(m3 * H.w, a3, v);
        return v;
      };
      float y, z = 0.f;
      if (from_parts) {
        if constexpr (BF16) y = fmaf(Hc.x, x_cur, acc_eff(Hc, accc, a1c, a2c, a3c));
        else next_input(P, Hc.x, fmaf(Hc.x, epsk, acc_eff(Hc, accc, a1c, a2c, a3c)), y, z);
      } else {
        y = fmaf(Hc.x, x_cur, acc_eff(Hc, accc, a1c, a2c, a3c));
        z = kTwoLog2e * y;
      }
      Hc = Hn; accc = accn; a1c = a1n; a2c = a2n; a3c = a3n;   // layer 2
      for (int l = 1;; ++l) {
        if constexpr (REC) if (act) a.rec[((size_t)(l - 1) * a.n_gen + (t - a.gen_base)) * y_stride + c_io] = y;
        if (l == M) break;
        {
          const int m = min(l + 2, M);   // two layers ahead (the last layers reload layer M: harmless)
          Hn = hv[(m - 1) * HV];
          accn = wcol[m * LS + o0];
          a1n = wcol[(m - 1) * LS + o1];
          a2n = wcol[(m - 1) * LS + o2];
          if constexpr (kChainLags >= 3) a3n = wcol[(m - 1) * LS + o3];
        }
        float av;
        if constexpr (BF16) {
          av = round_bf16(tanh_approx(y));
        } else {
          P = tanh_parts(y, z);
          av = tanh_value(P);
        }
        if (act) wcol[l * LS + o0] = av;
        if constexpr (BF16) y = fmaf(Hc.x, av, acc_eff(Hc, accc, a1c, a2c, a3c));
        else next_input(P, Hc.x, acc_eff(Hc, accc, a1c, a2c, a3c), y, z);
        Hc = Hn; accc = accn; a1c = a1n; a2c = a2n; a3c = a3n;
      }
      // y = y^M_t: hand the position to the tile warps, output, then the sampler
      // x_{t+1} = R(tanh(y) + eps_scale eps_t)
      {
        const int jp = r - r0;
        mbar_arrive(&act_ready[(jp % kRing) * CW + warp]);
      }
      if (act) a.y_out[(size_t)(t - a.gen_base) * y_stride + c_io] = y;
      const float epsv = ep[r * G + gg];
      float xn;
      if constexpr (BF16) {
        xn = round_bf16(tanh_approx(y) + a.eps_scale * epsv);
        x_cur = xn;
      } else {
        P = tanh_parts(y, z);
        epsk = a.eps_scale * epsv;
        xn = tanh_value(P) + epsk;
        x_cur = xn;
        from_parts = true;
      }
      // x_{t+1}; for the last position of the chunk it lands in the spare
      // position CH and goes to HBM with the write-back.
      if (act && t + 1 < g.L) wcol[(r + 1) * GP] = xn;
    }
  } else {
    // ---------------------------------------------------------------- tile warps
    // With a single chain warp, tile work stays off the scheduler that issues
    // for it (warp w issues on scheduler w % 4), so the latency-bound chain
    // shares its issue slots with no busy warp. With more chain warps every warp
    // takes pieces.
    const int nwarps = nt / 32;
    const bool spare_sched = CW == 1 && nwarps - CW > 4;
    auto is_tile = [&](int w) { return w >= CW && (!spare_sched || (w & 3) >= CW); };
    int tw = 0, ntw = 0;
    for (int w = CW; w < nwarps; ++w)
      if (is_tile(w)) {
        if (w < warp) ++tw;
        ++ntw;
      }
    if (is_tile(warp)) {
      // A row group k is (layer k / CW + 1, chain warp k % CW); this warp takes
      // k = tw, tw + ntw (two at a time when they share a chain warp), then
      // tw + 2 ntw, ... Everything about a row group but the step is resolved
      // once here for the first pair (the only one in most shapes), so a step
      // costs its waits and pieces alone.
      struct Grp {
        const float* src;
        float* dst;
        const float* taps;
        int c;
        bool act;
      };
      auto resolve = [&](int k) {
        Grp q;
        const int l = k / CW + 1;
        q.c = k - (l - 1) * CW;
        const int gg = q.c * 32 + lane;
        q.act = gg < Gc;
        const int ggs = q.act ? gg : 0;
        const int dl = (s0 + ggs) / g.B - d_lo;
        q.src = win + (l - 1) * LS + ggs;
        q.dst = win + l * LS + ggs;
        q.taps = tp + ((l - 1) * GdMax + dl) * TPS;
        return q;
      };
      const int MC = M * CW;
      const Grp gA0 = resolve(tw < MC ? tw : 0);
      const Grp gB0 = resolve(tw + ntw < MC ? tw + ntw : 0);
      for (int i = rs; i <= s_last; ++i) {
        // step i reads sources below i: position i-1 must be finished
        const int e0 = a.tab.first[i], e1 = a.tab.first[i + 1];
        const int j = i - rs, jp = i - 1 - r0;
        for (int k = tw; k < MC; k += 2 * ntw) {
          const int kB = k + ntw;
          const Grp gA = k == tw ? gA0 : resolve(k);
          const bool hasB = kB < MC;
          const Grp gB = !hasB ? gA : (k == tw ? gB0 : resolve(kB));
          const bool two = hasB && gB.c == gA.c;
          if (jp >= 0 && ok)
            ok = mbar_wait(&act_ready[(jp % kRing) * CW + gA.c], (jp / kRing) & 1, err, false, a.wait_limit);
          if (gA.act) {
            if (two) {
              for (int e = e0; e < e1; ++e) run_piece2(a.tab.e[e], gA.src, gA.dst, gA.taps, gB.src, gB.dst, gB.taps, GP);
            } else {
              for (int e = e0; e < e1; ++e) run_piece(a.tab.e[e], gA.src, gA.dst, gA.taps, GP);
            }
          }
          mbar_arrive(&tile_done[(j % kRing) * CW + gA.c]);
          if (two) {
            mbar_arrive(&tile_done[(j % kRing) * CW + gA.c]);
          } else if (hasB) {
            // the second row group belongs to another chain warp: on its own
            if (jp >= 0 && ok)
              ok = mbar_wait(&act_ready[(jp % kRing) * CW + gB.c], (jp / kRing) & 1, err, false, a.wait_limit);
            if (gB.act)
              for (int e = e0; e < e1; ++e) run_piece(a.tab.e[e], gB.src, gB.dst, gB.taps, GP);
            mbar_arrive(&tile_done[(j % kRing) * CW + gB.c]);
          }
        }
      }
    }
  }
  __syncthreads();

  // ---------------------------------------------------------------- write-back
  // The next chunk's first token, then positions [p0, c+CH) of layers 0..M-1:
  // new tokens and activations below p1, accumulators (including the on-chip
  // blocks' partial sums) from p1 on. Layer M's slots below p1 were consumed and
  // nothing reads them again; its accumulators from p1 on are still needed.
  if (r1 == CH && a.c + CH < g.L && tid < Gc) a.state[slot_index(g, 0, s0 + tid, a.c + CH)] = win[CH * GP + tid];
  const int re = min(CH, g.L - a.c);
  if (r0 == 0 && (re & 3) == 0 && (r1 & 3) == 0) {
    // one warp per layer: layers 0..M-1 from position 0, layer M from p1
    const int vpr = re >> 2;
    const int lv = 31 - __clz(vpr);
    const int wid = tid >> 5, lid = tid & 31, nw = nt >> 5;
    for (int l = wid; l <= M; l += nw) {
      const int j0 = l == M ? (r1 >> 2) : 0;
      const int nk = Gc << lv;
      for (int k = lid; k < nk; k += 32) {
        const int row = k >> lv, j = k & (vpr - 1);
        if (j < j0) continue;
        const float* w = win + l * LS + 4 * j * GP + row;
        *reinterpret_cast<float4*>(a.state + slot_index(g, l, s0 + row, a.c + 4 * j)) =
            make_float4(w[0], w[GP], w[2 * GP], w[3 * GP]);
      }
    }
  } else {
    for (int idx = tid; idx < (M + 1) * Gc * CH; idx += nt) {
      const int row = idx / CH, r = idx - row * CH;
      const int l = row / Gc, gg = row - l * Gc;
      const int rb = l == M ? r1 : r0;
      if (r >= rb && r < re) a.state[slot_index(g, l, s0 + gg, a.c + r)] = win[l * LS + r * GP + gg];
    }
  }
}

size_t chunk_smem_bytes(const Dims& g, int chunk, int G) { return chunk_shape(g, chunk, G).total * sizeof(float); }

// Warps per CTA: the chain warps, then enough warps for one tile warp per row
// group (layer, chain warp) up to the CTA's limit. With a single chain warp and
// more than four warps the kernel leaves scheduler 0 to the chain (warps
// 4, 8, 12 take no tile work), so those warps are added on top.
static int chunk_threads(const Dims& g, int G) {
  const int cw = (G + 31) / 32, max_w = kChunkMaxThreads / 32;
  const int want = g.M * cw;
  if (cw == 1) {
    int nw = 1, tiles = 0;
    while (tiles < want && nw < max_w) {
      if ((nw & 3) != 0) ++tiles;
      ++nw;
    }
    if (nw - cw <= 4) return 32 * (cw + (want < max_w - cw ? want : max_w - cw));   // no spare scheduler
    return 32 * nw;
  }
  return 32 * (cw + (want < max_w - cw ? want : max_w - cw));
}

bool chunk_cta_fills_sm(const Dims& g, int streams_per_cta) {
  return chunk_threads(g, streams_per_cta) >= kChunkMaxThreads;
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

using ChunkKernel = void (*)(Dims, ChunkArgs, int);
static ChunkKernel chunk_variant(bool bf16, bool rec, bool trig) {
  if (bf16) {
    if (rec) return trig ? k_chunk<true, true, true> : k_chunk<true, true, false>;
    return trig ? k_chunk<true, false, true> : k_chunk<true, false, false>;
  }
  if (rec) return trig ? k_chunk<false, true, true> : k_chunk<false, true, false>;
  return trig ? k_chunk<false, false, true> : k_chunk<false, false, false>;
}

cudaError_t configure_chunk(size_t smem) {
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  cudaError_t e = cudaSuccess;
  for (int v = 0; v < 8 && e == cudaSuccess; ++v) e = raise_smem_cap(chunk_variant(v & 1, v & 2, v & 4), smem);
  return e;
}

cudaError_t launch_chunk(const Dims& g, const ChunkArgs& a_in, int G, cudaStream_t st) {
  if (a_in.chunk < 2 || (a_in.chunk & (a_in.chunk - 1)) || a_in.chunk > kChunkMaxSteps) return cudaErrorInvalidValue;
  ChunkArgs a = a_in;
  // A launch over a whole chunk runs the re-timed pieces; one over part of a
  // chunk keeps the page's blocks, so the state at a call boundary is canonical.
  const bool whole = a.p0 == a.c && a.p1 == a.c + a.chunk;
  if (!build_chunk_table(a.chunk, whole, &a.tab, g.M <= kCoarseMaxLayers)) return cudaErrorInvalidValue;
  const size_t smem = chunk_smem_bytes(g, a.chunk, G);
  const int blocks = (g.S + G - 1) / G;
  const int nt = chunk_threads(g, G);
  // programmatic stream serialization: the launch may begin while the block
  // kernel before it drains (the kernel waits for it before reading the state)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)blocks);
  cfg.blockDim = dim3((unsigned)nt);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (g.bf16) {
    return cudaLaunchKernelEx(&cfg, chunk_variant(true, a.rec != nullptr, a.trigger != 0), g, a, G);
  }
  return cudaLaunchKernelEx(&cfg, chunk_variant(false, a.rec != nullptr, a.trigger != 0), g, a, G);
}

}  // namespace fi
