// FFT blocks (Lemma 1 and the circular-convolution trick of the Flash Inference
// summary page, "Punti di Innovazione Tecnica" 3) and the filter spectra
// ("Precomputazione FFT").
//
// A block of side U at step i adds sum_{s in [i-U, i)} h[t-s] a[s] to every
// target t in [i, i+U). With xx = [a[i-U..i) || 0_U] and hh = h[0..2U), the
// length-2U circular convolution xx (*) hh equals that sum at indices [U, 2U),
// so one real FFT of length 2U, a product with the precomputed spectrum of
// h[0..2U) and one inverse real FFT give the block.
//
// Real FFTs of length 2N (N = U) run as complex FFTs of N points on
// z[m] = x[2m] + i x[2m+1], followed by the usual split:
//   E[k] = (Z[k] + conj Z[N-k]) / 2,  O[k] = -i (Z[k] - conj Z[N-k]) / 2,
//   X[k] = E[k] + W_{2N}^k O[k],      X[N-k] = conj(E[k] - W_{2N}^k O[k]).
// The inverse packs Y = X * H back into N points,
//   Z'[k] = (Y[k] + conj Y[N-k]) + i (Y[k] - conj Y[N-k]) conj(W_{2N}^k),
// whose inverse complex FFT carries 2N * (y[2m] + i y[2m+1]); the 1/(2N) is
// folded into the stored spectrum. Zero padding means z[m] = 0 for m >= N/2,
// and only y[N..2N) (m >= N/2) is kept.
#include "fi_internal.cuh"
#include "fft.cuh"

namespace fi {

// W_{2N}^k = exp(-i pi k / N) (0 <= k <= N/2) for the split and pack of a real FFT
// of length 2N: from the table where consecutive k are consecutive entries (N of
// 2^14 and 2^13), else from the hardware sine/cosine (absolute error about 2^-21),
// since a warp's table loads at a stride of 2^15/(2N) entries touch one sector each.
template <int N>
__device__ __forceinline__ float2 split_twiddle(const float2* __restrict__ tw, int k) {
  constexpr int twstep = kTwiddleN / (2 * N);
  if constexpr (twstep <= 2) {
    return __ldg(tw + k * twstep);
  } else {
    float sn, cs;
    __sincosf((float)k * (3.14159265358979323846f / (float)N), &sn, &cs);
    return make_float2(cs, -sn);
  }
}

// Spectrum split + product + inverse pack, in place on sm (N complex points).
// H: N+1 spectrum values. Threads [0, T) of the transform.
template <int N, int T>
__device__ __forceinline__ void spectral_product(float2* sm, int tid, const float2* __restrict__ H,
                                                 const float2* __restrict__ tw) {
#pragma unroll
  for (int k = tid; k <= N / 2; k += T) {
    const int kk = (N - k) & (N - 1);
    const float2 zk = sm[fft_pad<N, T>(k)], zn = sm[fft_pad<N, T>(kk)];
    const float2 E = make_float2(0.5f * (zk.x + zn.x), 0.5f * (zk.y - zn.y));
    const float2 O = make_float2(0.5f * (zk.y + zn.y), -0.5f * (zk.x - zn.x));
    const float2 W = split_twiddle<N>(tw, k);
    const float2 WO = cmul(W, O);
    const float2 Xk = cadd(E, WO);
    const float2 Xn = cconj(csub(E, WO));
    const float2 Yk = cmul(Xk, __ldg(H + k));
    const float2 Yn = cmul(Xn, __ldg(H + (N - k)));
    const float2 A = cadd(Yk, cconj(Yn));
    const float2 Bv = cmul(csub(Yk, cconj(Yn)), cconj(W));
    sm[fft_pad<N, T>(k)] = make_float2(A.x - Bv.y, A.y + Bv.x);
    if (k != 0 && k != N / 2) sm[fft_pad<N, T>(N - k)] = make_float2(A.x + Bv.y, -A.y + Bv.x);
  }
}

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(dst))),
               "l"(src)
               : "memory");
}

// The accumulators a block adds into travel to shared memory while the
// transforms run (16-byte asynchronous copies; the target is 16-byte aligned).
template <int N, int T>
__device__ __forceinline__ void stage_dst(float2* ds, int tid, bool active, const float2* __restrict__ dst,
                                          int overwrite) {
  if (active && !overwrite) {
    for (int q = tid; q < N / 4; q += T) cp_async16(ds + 2 * q, dst + 2 * q);
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// Forward transform of z[m] = (x[2m], x[2m+1]) for m < N/2 and zero above,
// its first pass read straight from HBM; the result is left in sm.
template <int N, int T, class Sync>
__device__ __forceinline__ void fwd_from_global(float2* sm, int tid, bool active, const float2* __restrict__ src,
                                                Sync sync) {
  using S = FftShape<N, T>;
  {
    constexpr int R = 1 << S::rb(0);
    float2 v[S::P];
#pragma unroll
    for (int k = 0; k < S::P / R; ++k) {
      const int j = tid + k * T;
#pragma unroll
      for (int r = 0; r < R; ++r)
        v[k * R + r] = (active && r < R / 2) ? src[j + r * (N / R)] : make_float2(0.f, 0.f);
    }
    pass_compute<N, T, false, 0>(v, tid);
    pass_store<N, T, 0>(sm, v, tid);
    sync();
  }
  smem_passes<N, T, false, S::rb(0), false>(sm, tid, sync);
}

// Inverse transform of the packed spectrum in sm, its last pass written straight
// to HBM: only outputs m >= N/2 (the block's targets) are kept, added to the
// staged accumulators (or stored, for the first block to reach them).
template <int N, int T, class Sync>
__device__ __forceinline__ void inv_to_global(float2* sm, const float2* ds, int tid, bool active,
                                              float2* __restrict__ dst, int overwrite, int w_min, Sync sync) {
  using S = FftShape<N, T>;
  smem_passes<N, T, true, 0, true>(sm, tid, sync);
  constexpr int DL = last_pass_done<N, T>();
  constexpr int R = 1 << S::rb(DL);
  float2 v[S::P];
  pass_load<N, T, DL>(sm, v, tid);
  pass_compute<N, T, true, DL>(v, tid);
  asm volatile("cp.async.wait_all;" ::: "memory");
  sync();
  if (active) {
#pragma unroll
    for (int k = 0; k < S::P / R; ++k) {
      const int j = tid + k * T;
#pragma unroll
      for (int r = R / 2; r < R; ++r) {
        const int m = j + r * (N / R) - N / 2;
        const float2 o = v[k * R + r];
        float2 val = o;
        if (!overwrite) {
          const float2 p = ds[m];
          val = make_float2(p.x + o.x, p.y + o.y);
        }
        // targets below w_min (relative to dst) are left alone: positions 2m, 2m+1
        if (2 * m >= w_min) dst[m] = val;
        else if (2 * m + 1 >= w_min) reinterpret_cast<float*>(dst)[2 * m + 1] = val.y;
      }
    }
  }
}

template <int N, int T, class Sync>
__device__ __forceinline__ void tile_fft_body(float2* sm, float2* ds, int tid, bool active, const float2* __restrict__ src,
                                              float2* __restrict__ dst, const float2* __restrict__ H,
                                              const float2* __restrict__ tw, int overwrite, int w_min, Sync sync) {
  stage_dst<N, T>(ds, tid, active, dst, overwrite);
  fwd_from_global<N, T>(sm, tid, active, src, sync);
  spectral_product<N, T>(sm, tid, H, tw);
  sync();
  inv_to_global<N, T>(sm, ds, tid, active, dst, overwrite, w_min, sync);
}

// ---------------------------------------------------------------------------
// Blocks wider than one transform (U = m*N, N the largest transform): split the
// sources into m sub-blocks S_j of N and the targets into m sub-blocks T_k. The
// pair (S_j, T_k) is a block of side N whose lags run over
// h[U + (k-j-1)N + 1 .. U + (k-j+1)N - 1], so with the spectra
// G_delta = rFFT_2N(h[U + (delta-1)N .. U + (delta+1)N)) / 2N, delta = k-j in
// [-(m-1), m-1], target T_k receives irFFT_2N(sum_j X_j * G_{k-j})[N..2N), where
// X_j = rFFT_2N([S_j || 0]). One forward transform per source sub-block goes to
// a scratch buffer; one inverse transform per target sub-block reads it.
// ---------------------------------------------------------------------------

// Half spectrum X[0..N] of the real sequence packed in sm, written to out.
template <int N, int T>
__device__ __forceinline__ void store_half_spectrum(const float2* sm, int tid, float2* __restrict__ out,
                                                    const float2* __restrict__ tw) {
  for (int k = tid; k <= N / 2; k += T) {
    const int kk = (N - k) & (N - 1);
    const float2 zk = sm[fft_pad<N, T>(k)], zn = sm[fft_pad<N, T>(kk)];
    const float2 E = make_float2(0.5f * (zk.x + zn.x), 0.5f * (zk.y - zn.y));
    const float2 O = make_float2(0.5f * (zk.y + zn.y), -0.5f * (zk.x - zn.x));
    const float2 WO = cmul(split_twiddle<N>(tw, k), O);
    out[k] = cadd(E, WO);
    if (k != N / 2) out[N - k] = cconj(csub(E, WO));
  }
}

// item = row * m + j; row = (l-1)*S + s.
template <int N>
__global__ void __launch_bounds__(fft_cta_threads(N))
k_part_fwd(Dims g, const float* __restrict__ state, float2* __restrict__ xs, const float2* __restrict__ tw, int i,
           int m) {
  constexpr int T = fft_threads(N), F = fft_per_cta(N);
  extern __shared__ float2 fsm[];
  const int sub = threadIdx.x / T, tid = threadIdx.x - sub * T;
  float2* sm = fsm + sub * fft_smem_elems(N);
  const long item = (long)blockIdx.x * F + sub;
  const bool active = item < (long)g.M * g.S * m;
  const long row = active ? item / m : 0;
  const int j = active ? (int)(item - row * m) : 0;
  const int l = (int)(row / g.S) + 1, s = (int)(row % g.S);
  const int U = m * N;
  const float2* src = reinterpret_cast<const float2*>(state + slot_index(g, l - 1, s, i - U + j * N));
  if constexpr (T <= 32) fwd_from_global<N, T>(sm, tid, active, src, SyncWarp());
  else fwd_from_global<N, T>(sm, tid, active, src, SyncBlock());
  if (active) store_half_spectrum<N, T>(sm, tid, xs + (size_t)item * (N + 1), tw);
}

// item = row * m + k: target sub-block k of the row.
template <int N>
__global__ void __launch_bounds__(fft_cta_threads(N))
k_part_inv(Dims g, float* __restrict__ state, const float2* __restrict__ xs, const float2* __restrict__ gspec,
           const float2* __restrict__ tw, int i, int m, int overwrite, int t_min) {
  pdl_launch_dependents();
  constexpr int T = fft_threads(N), F = fft_per_cta(N);
  extern __shared__ float2 fsm[];
  const int sub = threadIdx.x / T, tid = threadIdx.x - sub * T;
  float2* sm = fsm + sub * fft_smem_elems(N);
  float2* ds = fsm + F * fft_smem_elems(N) + sub * (N / 2);
  const long item = (long)blockIdx.x * F + sub;
  const bool active = item < (long)g.M * g.S * m;
  const long row = active ? item / m : 0;
  const int k = active ? (int)(item - row * m) : 0;
  const int l = (int)(row / g.S) + 1, s = (int)(row % g.S), d = s / g.B;
  float2* dst = reinterpret_cast<float2*>(state + slot_index(g, l, s, i + k * N));
  // segment spectra of this (layer, channel): [2m-1][N+1], delta = k - j at index delta + m - 1
  const float2* G = gspec + ((size_t)(l - 1) * g.D + d) * (2 * m - 1) * (N + 1);
  const float2* X = xs + (size_t)row * m * (N + 1);
  stage_dst<N, T>(ds, tid, active, dst, overwrite);
  for (int f = tid; f <= N / 2; f += T) {
    const int fn = N - f;
    float2 yf = make_float2(0.f, 0.f), yn = make_float2(0.f, 0.f);
    for (int j = 0; j < m; ++j) {
      const float2* Xj = X + (size_t)j * (N + 1);
      const float2* Gd = G + (size_t)(k - j + m - 1) * (N + 1);
      const float2 a = cmul(Xj[f], Gd[f]);
      const float2 b = cmul(Xj[fn], Gd[fn]);
      yf = cadd(yf, a);
      yn = cadd(yn, b);
    }
    const float2 W = split_twiddle<N>(tw, f);
    const float2 A = cadd(yf, cconj(yn));
    const float2 Bv = cmul(csub(yf, cconj(yn)), cconj(W));
    sm[fft_pad<N, T>(f & (N - 1))] = make_float2(A.x - Bv.y, A.y + Bv.x);
    if (f != 0 && f != N / 2) sm[fft_pad<N, T>(fn)] = make_float2(A.x + Bv.y, -A.y + Bv.x);
  }
  if constexpr (T <= 32) {
    __syncwarp();
    inv_to_global<N, T>(sm, ds, tid, active, dst, overwrite, t_min - (i + k * N), SyncWarp());
  } else {
    __syncthreads();
    inv_to_global<N, T>(sm, ds, tid, active, dst, overwrite, t_min - (i + k * N), SyncBlock());
  }
}

// One FFT block for every (layer, stream): item = (l-1)*S + s. T threads per
// transform, F = cta_threads / T transforms per CTA.
// PDLW: the variant launched programmatically, which waits for the launch
// before it; plain launches use the variant without the instruction.
template <int N, int T = fft_threads(N), bool PDLW = false>
__global__ void __launch_bounds__(T >= 128 ? T : 128)
k_tile_fft(Dims g, float* __restrict__ state, const float2* __restrict__ spec,
           const float2* __restrict__ tw, int i, int overwrite, int t_min) {
  pdl_launch_dependents();
  if constexpr (PDLW) pdl_wait_primary();   // sources and accumulators come from the launch before
  constexpr int F = T >= 128 ? 1 : 128 / T;
  extern __shared__ float2 fsm[];
  const int sub = threadIdx.x / T, tid = threadIdx.x - sub * T;
  float2* sm = fsm + sub * fft_smem_elems(N);
  float2* ds = fsm + F * fft_smem_elems(N) + sub * (N / 2);   // staged accumulators
  const long item = (long)blockIdx.x * F + sub;
  const long items = (long)g.M * g.S;
  const bool active = item < items;
  const int l = active ? (int)(item / g.S) + 1 : 1;
  const int s = active ? (int)(item % g.S) : 0;
  const int d = s / g.B;
  const float2* src = reinterpret_cast<const float2*>(state + slot_index(g, l - 1, s, i - N));
  float2* dst = reinterpret_cast<float2*>(state + slot_index(g, l, s, i));
  const float2* H = spec + ((size_t)(l - 1) * g.D + d) * (N + 1);
  if constexpr (T <= 32) tile_fft_body<N, T>(sm, ds, tid, active, src, dst, H, tw, overwrite, t_min - i, SyncWarp());
  else tile_fft_body<N, T>(sm, ds, tid, active, src, dst, H, tw, overwrite, t_min - i, SyncBlock());
}

// ---------------------------------------------------------------------------
// Paired FFT blocks (even batch): two sequences b, b+1 of one (layer, channel)
// share the filter, so their sources go into one complex sequence
// z[m] = x_b[m] + i x_{b+1}[m] (m < U, zero above) of N2 = 2U points. Its DFT is
// X_b + i X_{b+1}; multiplied by the filter's 2U-point spectrum H (the same
// spectrum for both, and H[2U-k] = conj H[k] because h is real) it becomes
// Y_b + i Y_{b+1}, whose inverse carries y_b in the real part and y_{b+1} in the
// imaginary part. The product is pointwise, so no real-FFT split is needed and
// the forward transform's last pass, the product and the inverse's first pass
// run on the same registers: the Stockham last pass leaves thread j holding
// points j + r N2/R, which is exactly what the inverse's first pass of the same
// radix reads (the inverse takes its passes in the opposite radix order).
// ---------------------------------------------------------------------------
template <int N2, int T, int PL = 0>
__device__ __forceinline__ void tile_fft2_body(float2* sm, float* ds, int tid, bool active,
                                               const float* __restrict__ src1, const float* __restrict__ src2,
                                               float* __restrict__ dst1, float* __restrict__ dst2,
                                               const float2* __restrict__ H,
                                               int overwrite, int w_min) {
  constexpr int U = N2 / 2;
  constexpr int SHF = PL << 4, SHI = (PL << 4) | 1;   // forward plan; the inverse takes it reversed
  using SF = FftShape<N2, T, SHF>;
  using SI = FftShape<N2, T, SHI>;
  auto sync = [] {
    if constexpr (T <= 32) __syncwarp();
    else __syncthreads();
  };
  // accumulators of both sequences travel to shared memory meanwhile
  if (active && !overwrite) {
    for (int q = tid; q < U / 4; q += T) {
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(ds + 4 * q))),
                   "l"(dst1 + 4 * q) : "memory");
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(static_cast<uint32_t>(__cvta_generic_to_shared(ds + U + 4 * q))),
                   "l"(dst2 + 4 * q) : "memory");
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
  float2 v[SF::P];
  {
    // forward pass 0 straight from HBM; points m >= U are the zero padding
    constexpr int R = 1 << SF::rb(0);
#pragma unroll
    for (int k = 0; k < SF::P / R; ++k) {
      const int j = tid + k * T;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int m = j + r * (N2 / R);
        v[k * R + r] = (active && r < R / 2) ? make_float2(__ldg(src1 + m), __ldg(src2 + m)) : make_float2(0.f, 0.f);
      }
    }
    pass_compute<N2, T, false, 0, SHF>(v, tid);
    if constexpr (!SF::last(0)) {
      pass_store<N2, T, 0, SHF>(sm, v, tid);
      sync();
      smem_passes<N2, T, false, SF::rb(0), true, SHF>(sm, tid, sync);
      constexpr int DL = last_pass_done<N2, T, 0, SHF>();
      pass_load<N2, T, DL, SHF>(sm, v, tid);
      pass_compute<N2, T, false, DL, SHF>(v, tid);
    }
  }
  {
    // spectrum product on the points this thread holds: j + r N2/R
    constexpr int R = 1 << SF::rb(last_pass_done<N2, T, 0, SHF>());
    static_assert(R == (1 << SI::rb(0)), "inverse must start with the forward's last radix");
#pragma unroll
    for (int k = 0; k < SF::P / R; ++k) {
      const int j = tid + k * T;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int kk = j + r * (N2 / R);
        float2 h = __ldg(H + (kk <= U ? kk : N2 - kk));
        if (kk > U) h.y = -h.y;
        v[k * R + r] = cmul(v[k * R + r], h);
      }
    }
  }
  // inverse, first pass in registers
  pass_compute<N2, T, true, 0, SHI>(v, tid);
  if constexpr (!SI::last(0)) {
    sync();   // every thread is done reading sm in the forward's last pass
    pass_store<N2, T, 0, SHI>(sm, v, tid);
    sync();
    smem_passes<N2, T, true, SI::rb(0), true, SHI>(sm, tid, sync);
    constexpr int DL = last_pass_done<N2, T, 0, SHI>();
    pass_load<N2, T, DL, SHI>(sm, v, tid);
    pass_compute<N2, T, true, DL, SHI>(v, tid);
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  sync();
  if (active) {
    constexpr int R = 1 << SI::rb(last_pass_done<N2, T, 0, SHI>());
#pragma unroll
    for (int k = 0; k < SI::P / R; ++k) {
      const int j = tid + k * T;
#pragma unroll
      for (int r = R / 2; r < R; ++r) {
        const int m = j + r * (N2 / R) - U;
        const float2 o = v[k * R + r];
        if (m < w_min) continue;
        if (overwrite) {
          dst1[m] = o.x;
          dst2[m] = o.y;
        } else {
          dst1[m] = ds[m] + o.x;
          dst2[m] = ds[U + m] + o.y;
        }
      }
    }
  }
}

// item = pair ((l-1)*S/2 + p): sequences s = 2p and 2p+1 (same channel, B even).
// CTAs per SM the paired blocks ask the compiler to fit (register budget),
// from a B200 sweep of 1..3 at the 18 x 3456-row batch: 3 for side 256
// (91 -> 74 us per launch), 2 for side 2048 (965 -> 730 us); more hurt the
// sides that hold 32 points per thread (8192: 4.1 -> 6.5 ms).
__host__ __device__ constexpr int fft2_min_blocks(int n2) { return n2 == 512 ? 3 : n2 == 4096 ? 2 : 1; }

template <int N2, int T, int PL = 0, bool PDLW = false>
__global__ void __launch_bounds__(T >= 128 ? T : 128, fft2_min_blocks(N2))
k_tile_fft2(Dims g, float* __restrict__ state, const float2* __restrict__ spec, int i,
            int overwrite, int t_min) {
  pdl_launch_dependents();
  if constexpr (PDLW) pdl_wait_primary();   // sources and accumulators come from the launch before
  constexpr int U = N2 / 2;
  constexpr int F = T >= 128 ? 1 : 128 / T;
  extern __shared__ float2 fsm[];
  const int sub = threadIdx.x / T, tid = threadIdx.x - sub * T;
  float2* sm = fsm + sub * fft_smem_elems(N2);
  float* ds = reinterpret_cast<float*>(fsm + F * fft_smem_elems(N2)) + sub * 2 * U;
  const long item = (long)blockIdx.x * F + sub;
  const int half = g.S / 2;
  const bool active = item < (long)g.M * half;
  const int l = active ? (int)(item / half) + 1 : 1;
  const int s1 = active ? 2 * (int)(item % half) : 0;
  const int d = s1 / g.B;
  const float* src1 = state + slot_index(g, l - 1, s1, i - U);
  const float* src2 = state + slot_index(g, l - 1, s1 + 1, i - U);
  float* dst1 = state + slot_index(g, l, s1, i);
  float* dst2 = state + slot_index(g, l, s1 + 1, i);
  const float2* H = spec + ((size_t)(l - 1) * g.D + d) * (U + 1);
  tile_fft2_body<N2, T, PL>(sm, ds, tid, active, src1, src2, dst1, dst2, H, overwrite, t_min - i);
}

// ---------------------------------------------------------------------------
// Prompt prefill (summary page, Limitazioni 4, "Fase di Prompt": the prompt's
// positions are all known, so each layer is one offline causal convolution).
// For a prompt of p <= N positions (N a power of two), y^l_t for t < p is the
// causal convolution of a^{l-1}_0..p-1 with h^l, computed by one real FFT of
// length 2N against the spectrum of h[0..N) zero-padded to 2N: both sequences
// have support [0, N), so the circular convolution of length 2N has no
// wrap-around and its first N outputs are the causal convolution (lag 0, the
// red cell, included). One launch per layer, one transform per stream; the
// block (tanh, bf16 rounding) is applied on the way out.
// ---------------------------------------------------------------------------
template <int N, int T = fft_threads(N)>
__global__ void __launch_bounds__(T >= 128 ? T : 128)
k_prefix_conv(Dims g, float* __restrict__ state, const float2* __restrict__ spec, const float2* __restrict__ tw,
              int l, int p, float* __restrict__ y_out, float* __restrict__ rec, int n_rec) {
  constexpr int F = T >= 128 ? 1 : 128 / T;
  using S = FftShape<N, T>;
  extern __shared__ float2 fsm[];
  const int sub = threadIdx.x / T, tid = threadIdx.x - sub * T;
  float2* sm = fsm + sub * fft_smem_elems(N);
  const long item = (long)blockIdx.x * F + sub;
  const bool active = item < g.S;
  const int s = active ? (int)item : 0, d = s / g.B, b = s - d * g.B;
  const float* src = state + slot_index(g, l - 1, s, 0);
  const float2* H = spec + ((size_t)(l - 1) * g.D + d) * (N + 1);
  auto sync = [] {
    if constexpr (T <= 32) __syncwarp();
    else __syncthreads();
  };
  {
    // forward pass 0 from HBM: z[m] = (a[2m], a[2m+1]), zero at positions >= p
    constexpr int R = 1 << S::rb(0);
    float2 v[S::P];
#pragma unroll
    for (int k = 0; k < S::P / R; ++k) {
      const int j = tid + k * T;
#pragma unroll
      for (int r = 0; r < R; ++r) {
        const int t0 = 2 * (j + r * (N / R));
        v[k * R + r] = (active && r < R / 2)
                           ? make_float2(t0 < p ? src[t0] : 0.f, t0 + 1 < p ? src[t0 + 1] : 0.f)
                           : make_float2(0.f, 0.f);
      }
    }
    pass_compute<N, T, false, 0>(v, tid);
    pass_store<N, T, 0>(sm, v, tid);
    sync();
  }
  smem_passes<N, T, false, S::rb(0), false>(sm, tid, sync);
  spectral_product<N, T>(sm, tid, H, tw);
  sync();
  smem_passes<N, T, true, 0, true>(sm, tid, sync);
  constexpr int DL = last_pass_done<N, T>();
  constexpr int R = 1 << S::rb(DL);
  float2 v[S::P];
  pass_load<N, T, DL>(sm, v, tid);
  pass_compute<N, T, true, DL>(v, tid);
  if (!active) return;
  const size_t io = (size_t)b * g.D + d;
  float* dst = state + slot_index(g, l, s, 0);
#pragma unroll
  for (int k = 0; k < S::P / R; ++k) {
    const int j = tid + k * T;
#pragma unroll
    for (int r = 0; r < R / 2; ++r) {
      const int t0 = 2 * (j + r * (N / R));
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int t = t0 + q;
        if (t >= p) continue;
        const float y = q ? v[k * R + r].y : v[k * R + r].x;
        if (rec) rec[((size_t)(l - 1) * n_rec + t) * g.S + io] = y;
        if (l < g.M) dst[t] = round_act(tanhf(y), g.bf16);
        else if (y_out) y_out[(size_t)t * g.S + io] = y;
      }
    }
  }
}

// Prompt tokens x[t][b][d] into the layer-0 slots.
__global__ void k_store_tokens(Dims g, float* __restrict__ state, const void* __restrict__ x, int p) {
  const size_t total = (size_t)p * g.S;
  for (size_t k = (size_t)blockIdx.x * blockDim.x + threadIdx.x; k < total; k += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(k / g.S);
    const int r = (int)(k - (size_t)t * g.S);   // r = b*D + d
    const int b = r / g.D, d = r - b * g.D;
    state[slot_index(g, 0, d * g.B + b, t)] = round_act(load_token(x, k, g.bf16), g.bf16);
  }
}

// Spectrum of h[0..2N) / (2N) for one (layer, channel): item = l*D + d.
template <int N>
__global__ void __launch_bounds__(fft_cta_threads(N))
k_spectra(Dims g, const float* __restrict__ taps, float2* __restrict__ spec, const float2* __restrict__ tw, int off,
          int nseg, int seg0, int pad) {
  constexpr int T = fft_threads(N), F = fft_per_cta(N);
  constexpr int twstep = kTwiddleN / (2 * N);
  extern __shared__ float2 fsm[];
  const int sub = threadIdx.x / T, tid = threadIdx.x - sub * T;
  float2* sm = fsm + sub * fft_smem_elems(N);
  // item = (l*D + d)*nseg + segment; segment e reads h[off + (seg0+e)*N .. + 2N)
  const long item = (long)blockIdx.x * F + sub;
  const bool active = item < (long)g.M * g.D * nseg;
  const long ld = active ? item / nseg : 0;
  const int e = active ? (int)(item - ld * nseg) : 0;
  const float2* src = reinterpret_cast<const float2*>(taps + (size_t)ld * g.L + off + (size_t)(seg0 + e) * N);
  // pad: only h[0..N) (complex points m < N/2), zero above
  for (int m = tid; m < N; m += T)
    sm[fft_pad<N, T>(m)] = (active && (!pad || m < N / 2)) ? src[m] : make_float2(0.f, 0.f);
  if constexpr (T <= 32) {
    __syncwarp();
    fft_smem<N, T, false>(sm, tid, SyncWarp());
  } else {
    __syncthreads();
    fft_smem<N, T, false>(sm, tid, SyncBlock());
  }
  if (!active) return;
  float2* H = spec + (size_t)item * (N + 1);
  const float scale = 1.0f / (2.0f * N);
  for (int k = tid; k <= N / 2; k += T) {
    const int kk = (N - k) & (N - 1);
    const float2 zk = sm[fft_pad<N, T>(k)], zn = sm[fft_pad<N, T>(kk)];
    const float2 E = make_float2(0.5f * (zk.x + zn.x), 0.5f * (zk.y - zn.y));
    const float2 O = make_float2(0.5f * (zk.y + zn.y), -0.5f * (zk.x - zn.x));
    const float2 WO = cmul(__ldg(tw + k * twstep), O);
    H[k] = cscale(cadd(E, WO), scale);
    if (k != N / 2) H[N - k] = cscale(cconj(csub(E, WO)), scale);
  }
}

template <int N>
__global__ void __launch_bounds__(fft_cta_threads(N))
k_debug_fft(int count, const float2* __restrict__ in, float2* __restrict__ out, int inverse) {
  constexpr int T = fft_threads(N), F = fft_per_cta(N);
  extern __shared__ float2 fsm[];
  const int sub = threadIdx.x / T, tid = threadIdx.x - sub * T;
  float2* sm = fsm + sub * fft_smem_elems(N);
  const long item = (long)blockIdx.x * F + sub;
  const bool active = item < count;
  for (int m = tid; m < N; m += T) sm[fft_pad<N, T>(m)] = active ? in[item * N + m] : make_float2(0.f, 0.f);
  if constexpr (T <= 32) {
    __syncwarp();
    if (inverse) fft_smem<N, T, true>(sm, tid, SyncWarp());
    else fft_smem<N, T, false>(sm, tid, SyncWarp());
  } else {
    __syncthreads();
    if (inverse) fft_smem<N, T, true>(sm, tid, SyncBlock());
    else fft_smem<N, T, false>(sm, tid, SyncBlock());
  }
  if (!active) return;
  for (int m = tid; m < N; m += T) out[item * N + m] = sm[fft_pad<N, T>(m)];
}

// ------------------------------------------------------------------ dispatch
// Block launches with pdl allow programmatic stream serialization: the grid
// may be launched while the chunk kernel before it finishes (its CTAs wait for
// it with pdl_wait_primary before reading the state).
static cudaLaunchConfig_t pdl_config(cudaLaunchAttribute (&attr)[1], unsigned blocks, int threads, size_t smem,
                                     cudaStream_t st) {
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(blocks);
  cfg.blockDim = dim3((unsigned)threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cfg;
}

template <int N>
static size_t fft_smem_bytes() { return (size_t)fft_per_cta(N) * fft_smem_elems(N) * sizeof(float2); }

template <class K>
static cudaError_t prepare(K kernel, size_t smem) {
  if (smem > 48 * 1024) return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  return cudaSuccess;
}

template <int N, int T = fft_threads(N)>
static cudaError_t tile_fft_n(const Dims& g, float* state, const float2* spec, const float2* tw, int i,
                              int t_min, cudaStream_t st, bool pdl) {
  constexpr int F = T >= 128 ? 1 : 128 / T;
  const size_t smem = (size_t)F * (fft_smem_elems(N) + N / 2) * sizeof(float2);
  cudaError_t e = pdl ? prepare(k_tile_fft<N, T, true>, smem) : prepare(k_tile_fft<N, T, false>, smem);
  if (e != cudaSuccess) return e;
  const long items = (long)g.M * g.S;
  const long blocks = (items + F - 1) / F;
  const int overwrite = is_pow2(i) ? 1 : 0;
  if (!pdl) {   // the plain launch costs the host less (launch-bound stacks)
    k_tile_fft<N, T, false><<<(unsigned)blocks, T * F, smem, st>>>(g, state, spec, tw, i, overwrite, t_min);
    return cudaGetLastError();
  }
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pdl_config(attr, (unsigned)blocks, T * F, smem, st);
  return cudaLaunchKernelEx(&cfg, k_tile_fft<N, T, true>, g, state, spec, tw, i, overwrite, t_min);
}

// Points per thread of the paired blocks (N2 = 2U points per pair): the choice
// that avoids a radix-2 pass (radix 32 where log2 N2 = 9, 10, 13, 14; radix 16
// where it is 7, 8, 11, 12).
__host__ __device__ constexpr int fft2_points(int n2) {
  return (n2 == 512 || n2 == 1024 || n2 == 8192 || n2 == 16384) ? 32 : 16;
}
// Pass plan of the paired blocks (FftShape's PL; 0 = radix min(32, P) passes).
__host__ __device__ constexpr int fft2_plan(int /*n2*/) { return 0; }

template <int N2, int P = fft2_points(N2), int PL = fft2_plan(N2)>
static cudaError_t tile_fft2_n(const Dims& g, float* state, const float2* spec, const float2* tw, int i,
                               int t_min, cudaStream_t st, bool pdl) {
  constexpr int T = N2 / P;
  constexpr int F = T >= 128 ? 1 : 128 / T;
  const size_t smem = (size_t)F * (fft_smem_elems(N2) * sizeof(float2) + (size_t)N2 * sizeof(float));
  cudaError_t e = pdl ? prepare(k_tile_fft2<N2, T, PL, true>, smem) : prepare(k_tile_fft2<N2, T, PL, false>, smem);
  if (e != cudaSuccess) return e;
  const long items = (long)g.M * (g.S / 2);
  const long blocks = (items + F - 1) / F;
  const int overwrite = is_pow2(i) ? 1 : 0;
  if (!pdl) {   // the plain launch costs the host less (launch-bound stacks)
    k_tile_fft2<N2, T, PL, false><<<(unsigned)blocks, T * F, smem, st>>>(g, state, spec, i, overwrite, t_min);
    return cudaGetLastError();
  }
  cudaLaunchAttribute attr[1];
  cudaLaunchConfig_t cfg = pdl_config(attr, (unsigned)blocks, T * F, smem, st);
  return cudaLaunchKernelEx(&cfg, k_tile_fft2<N2, T, PL, true>, g, state, spec, i, overwrite, t_min);
}

template <int N>
static cudaError_t spectra_n(const Dims& g, const float* taps, float2* spec, const float2* tw, int nseg,
                             cudaStream_t st, int pad = 0) {
  const size_t smem = fft_smem_bytes<N>();
  cudaError_t e = prepare(k_spectra<N>, smem);
  if (e != cudaSuccess) return e;
  const long items = (long)g.M * g.D * nseg;
  const long blocks = (items + fft_per_cta(N) - 1) / fft_per_cta(N);
  k_spectra<N><<<(unsigned)blocks, fft_cta_threads(N), smem, st>>>(g, taps, spec, tw, 0, nseg, 0, pad);
  return cudaGetLastError();
}

template <int N>
static cudaError_t debug_fft_n(int count, const float2* in, float2* out, int inverse, const float2* tw,
                               cudaStream_t st) {
  const size_t smem = fft_smem_bytes<N>();
  cudaError_t e = prepare(k_debug_fft<N>, smem);
  if (e != cudaSuccess) return e;
  const long blocks = ((long)count + fft_per_cta(N) - 1) / fft_per_cta(N);
  k_debug_fft<N><<<(unsigned)blocks, fft_cta_threads(N), smem, st>>>(count, in, out, inverse);
  return cudaGetLastError();
}

#define FI_FFT_SWITCH(q, CALL)            \
  switch (q) {                            \
    case 6: return CALL(64);              \
    case 7: return CALL(128);             \
    case 8: return CALL(256);             \
    case 9: return CALL(512);             \
    case 10: return CALL(1024);           \
    case 11: return CALL(2048);           \
    case 12: return CALL(4096);           \
    case 13: return CALL(8192);           \
    case 14: return CALL(16384);          \
    default: return cudaErrorInvalidValue; \
  }

cudaError_t launch_tile_fft(const Dims& g, float* state, const float2* spectrum_q, const float2* twiddle, int i,
                            int t_min, cudaStream_t st, bool pdl) {
  const int U = i & -i;
  const int q = ilog2((uint32_t)U);
  if (g.B % 2 == 0 && q <= kMaxFftLog2 - 1) {
    // two sequences of a channel per complex transform of 2U points
#define CALL(n) tile_fft2_n<2 * (n)>(g, state, spectrum_q, twiddle, i, t_min, st, pdl)
    switch (q) {
      case 6: return CALL(64);
      case 7: return CALL(128);
      case 8: return CALL(256);
      case 9: return CALL(512);
      case 10: return CALL(1024);
      case 11: return CALL(2048);
      case 12: return CALL(4096);
      case 13: return CALL(8192);
      default: return cudaErrorInvalidValue;
    }
#undef CALL
  }
#define CALL(n) tile_fft_n<n>(g, state, spectrum_q, twiddle, i, t_min, st, pdl)
  FI_FFT_SWITCH(q, CALL)
#undef CALL
}

cudaError_t launch_spectra(const Dims& g, const float* taps, float2* spectrum_q, const float2* twiddle, int q,
                           cudaStream_t st) {
#define CALL(n) spectra_n<n>(g, taps, spectrum_q, twiddle, 1, st)
  FI_FFT_SWITCH(q, CALL)
#undef CALL
}

cudaError_t launch_part_spectra(const Dims& g, const float* taps, float2* gspec, const float2* twiddle, int m,
                                cudaStream_t st) {
  return spectra_n<1 << kMaxFftLog2>(g, taps, gspec, twiddle, 2 * m - 1, st);
}

cudaError_t launch_part_block(const Dims& g, float* state, float2* xs, const float2* gspec, const float2* twiddle,
                              int i, int t_min, cudaStream_t st) {
  constexpr int N = 1 << kMaxFftLog2;
  const int m = (i & -i) / N;
  const long items = (long)g.M * g.S * m;
  const long blocks = (items + fft_per_cta(N) - 1) / fft_per_cta(N);
  size_t smem = fft_smem_bytes<N>();
  cudaError_t e = prepare(k_part_fwd<N>, smem);
  if (e != cudaSuccess) return e;
  k_part_fwd<N><<<(unsigned)blocks, fft_cta_threads(N), smem, st>>>(g, state, xs, twiddle, i, m);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  smem += (size_t)fft_per_cta(N) * (N / 2) * sizeof(float2);
  if ((e = prepare(k_part_inv<N>, smem)) != cudaSuccess) return e;
  k_part_inv<N><<<(unsigned)blocks, fft_cta_threads(N), smem, st>>>(g, state, xs, gspec, twiddle, i, m,
                                                                   is_pow2(i) ? 1 : 0, t_min);
  return cudaGetLastError();
}

cudaError_t launch_debug_fft(int log2n, int count, const float2* in, float2* out, int inverse,
                             const float2* twiddle, cudaStream_t st) {
#define CALL(n) debug_fft_n<n>(count, in, out, inverse, twiddle, st)
  FI_FFT_SWITCH(log2n, CALL)
#undef CALL
}

template <int N>
static cudaError_t prefix_n(const Dims& g, float* state, const float* taps, float2* spec, const float2* tw, int p,
                            const void* x, float* y_out, float* rec, cudaStream_t st) {
  cudaError_t e = spectra_n<N>(g, taps, spec, tw, 1, st, 1);
  if (e != cudaSuccess) return e;
  k_store_tokens<<<148 * 4, 256, 0, st>>>(g, state, x, p);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  constexpr int T = fft_threads(N), F = T >= 128 ? 1 : 128 / T;
  const size_t smem = (size_t)F * fft_smem_elems(N) * sizeof(float2);
  if ((e = prepare(k_prefix_conv<N>, smem)) != cudaSuccess) return e;
  const long blocks = ((long)g.S + F - 1) / F;
  for (int l = 1; l <= g.M; ++l) {
    k_prefix_conv<N><<<(unsigned)blocks, T * F, smem, st>>>(g, state, spec, tw, l, p, y_out, rec, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

int prefix_transform_log2(int p) {
  int q = kMinFftLog2;
  while ((1 << q) < p) ++q;
  return q;
}

cudaError_t launch_prefix(const Dims& g, float* state, const float* taps, float2* spec, const float2* twiddle, int p,
                          const void* x, float* y_out, float* rec, cudaStream_t st) {
  const int q = prefix_transform_log2(p);
#define CALL(n) prefix_n<n>(g, state, taps, spec, twiddle, p, x, y_out, rec, st)
  FI_FFT_SWITCH(q, CALL)
#undef CALL
}

}  // namespace fi
