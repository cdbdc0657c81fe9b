// Complex FFT of N = 2^k points held in shared memory, used by the FFT blocks
// (Lemma 1 of the Flash Inference summary page: tau by FFT) and by the filter
// spectrum precompute ("Precomputazione FFT").
//
// Formulation: Stockham autosort, decimation in time (Govindaraju et al.,
// "High Performance Discrete Fourier Transforms on Graphics Processors", SC'08):
// in pass s with radix R and Ns = product of the earlier radices, element j of
// N/R reads R values at stride N/R, multiplies value r by W_{Ns*R}^{r*(j mod Ns)},
// runs an R-point DFT in registers and writes value r to
// (j div Ns)*Ns*R + (j mod Ns) + r*Ns. The output is in natural order.
//
// T threads cooperate on one transform, each holding P = N/T points; the radix
// is min(32, P) (the last pass takes what is left). Each pass loads all of a
// thread's points, synchronises, then stores, so one buffer suffices. Shared
// memory indices are padded by one slot per 16 (idx + idx/16) so the stride-16
// stores of the first pass do not collide in the same bank.
#pragma once

#include <cuda_runtime.h>

#include <utility>

#include "fi_internal.cuh"

namespace fi {

// Shared-memory index of point i: one pad slot per 2^PADSHIFT points, with the
// span chosen so that the strided Stockham stores of a pass hit distinct banks
// (32 points per thread: one per 32; 16 or fewer: one per 16).
template <int N, int T>
__host__ __device__ constexpr int fft_pad(int i) { return i + (i >> ((N / T >= 32) ? 5 : 4)); }
// Upper bound of the padded length, for any thread count.
__host__ __device__ constexpr int fft_smem_elems(int n) { return n + (n >> 4); }
__host__ __device__ constexpr int clog2(int v) { return v <= 1 ? 0 : 1 + clog2(v >> 1); }
__host__ __device__ constexpr int cmin(int a, int b) { return a < b ? a : b; }

__device__ __forceinline__ float2 cadd(float2 a, float2 b) { return make_float2(a.x + b.x, a.y + b.y); }
__device__ __forceinline__ float2 csub(float2 a, float2 b) { return make_float2(a.x - b.x, a.y - b.y); }
__device__ __forceinline__ float2 cconj(float2 a) { return make_float2(a.x, -a.y); }
__device__ __forceinline__ float2 cscale(float2 a, float s) { return make_float2(a.x * s, a.y * s); }
__device__ __forceinline__ float2 cmul(float2 a, float2 b) {
  return make_float2(fmaf(a.x, b.x, -a.y * b.y), fmaf(a.x, b.y, a.y * b.x));
}
// multiply by i and by -i
__device__ __forceinline__ float2 cmul_i(float2 a) { return make_float2(-a.y, a.x); }
__device__ __forceinline__ float2 cmul_mi(float2 a) { return make_float2(a.y, -a.x); }

// cos of 2*pi*m/32 for m in [0, 32), by quadrant symmetry from the first
// quadrant's values (decimal expansions of the constants).
__host__ __device__ constexpr float cos32(int m) {
  constexpr float q[9] = {1.0f,
                          0.98078528040323044913f,   // cos(pi/16)
                          0.92387953251128675613f,   // cos(pi/8)
                          0.83146961230254523708f,   // cos(3pi/16)
                          0.70710678118654752440f,   // cos(pi/4)
                          0.55557023301960222474f,   // cos(5pi/16)
                          0.38268343236508977173f,   // cos(3pi/8)
                          0.19509032201612826785f,   // cos(7pi/16)
                          0.0f};
  m &= 31;
  return m <= 8 ? q[m] : m <= 16 ? -q[16 - m] : m <= 24 ? -q[m - 16] : q[32 - m];
}
__host__ __device__ constexpr float sin32(int m) { return cos32(m - 8); }  // sin x = cos(x - pi/2)

// v * W_32^m where W_32 = exp(-2 pi i / 32) (forward) or its conjugate (inverse).
// m is a compile-time constant after unrolling, so the branches fold away.
template <bool INV>
__device__ __forceinline__ float2 mul_w32(float2 v, int m) {
  m &= 31;
  if (m == 0) return v;
  if (m == 16) return make_float2(-v.x, -v.y);
  if (m == 8) return INV ? cmul_i(v) : cmul_mi(v);
  if (m == 24) return INV ? cmul_mi(v) : cmul_i(v);
  const float c = cos32(m);
  const float s = INV ? sin32(m) : -sin32(m);
  return cmul(v, make_float2(c, s));
}

__host__ __device__ constexpr int bitrev(int x, int bits) {
  return bits == 0 ? 0 : ((x & 1) << (bits - 1)) | bitrev(x >> 1, bits - 1);
}
template <int K, int BITS>
constexpr int kBitrev = bitrev(K, BITS);

// v[k] = t[bitrev(k)] with every index a template constant.
template <int BITS, int... K>
__device__ __forceinline__ void bitrev_copy(float2* v, const float2* t, std::integer_sequence<int, K...>) {
  ((v[K] = t[kBitrev<K, BITS>]), ...);
}

// One decimation-in-frequency stage of butterflies with half-span SPAN, then the
// next stage (template recursion keeps every index a compile-time constant).
template <int R, int SPAN, bool INV>
__device__ __forceinline__ void dif_stage(float2* v) {
#pragma unroll
  for (int g0 = 0; g0 < R; g0 += 2 * SPAN) {
#pragma unroll
    for (int j = 0; j < SPAN; ++j) {
      const float2 a = v[g0 + j], b = v[g0 + j + SPAN];
      v[g0 + j] = cadd(a, b);
      v[g0 + j + SPAN] = mul_w32<INV>(csub(a, b), j * (32 / (2 * SPAN)));
    }
  }
  if constexpr (SPAN > 1) dif_stage<R, SPAN / 2, INV>(v);
}

// R-point DFT of v[0..R) in registers (R = 2, 4, 8, 16 or 32): decimation in
// frequency, then a fixed permutation undoes the bit reversal.
template <int R, bool INV>
__device__ __forceinline__ void dft_reg(float2* v) {
  constexpr int B = clog2(R);
  dif_stage<R, R / 2, INV>(v);
  float2 t[R];
#pragma unroll
  for (int k = 0; k < R; ++k) t[k] = v[k];
  bitrev_copy<B>(v, t, std::make_integer_sequence<int, R>{});
}

struct SyncWarp { __device__ __forceinline__ void operator()() const { __syncwarp(); } };
struct SyncBlock { __device__ __forceinline__ void operator()() const { __syncthreads(); } };

// v[r] *= w^r for r = 1..R-1 (w = W_{NSR}^{kk}, NSR = Ns R, forward sign;
// conjugated for the inverse). w, w^4, w^8 (and w^16) come from the hardware
// sine/cosine (__sincosf, absolute error about 2^-21 on [-pi, pi]) with the angle
// reduced to that range; the other powers are products of at most four of them.
// Measured on B200, this beats loading the four values from a table by 9-19 % per
// FFT block: the table loads of a pass are strided over a 256 KB table, so each
// warp load touched 16-32 sectors.
template <int R, int NSR, bool INV>
__device__ __forceinline__ void apply_twiddles(float2* v, int kk) {
  auto ld = [&](int r) {
    int m = r * kk;                        // in [0, NSR)
    if (2 * m > NSR) m -= NSR;             // angle in (-pi, pi]
    float sn, cs;
    __sincosf((float)m * (-6.28318530717958647692f / (float)NSR), &sn, &cs);
    return make_float2(cs, INV ? -sn : sn);
  };
  const float2 w1 = ld(1);
  v[1] = cmul(v[1], w1);
  if constexpr (R == 2) return;
  const float2 w2 = cmul(w1, w1);
  const float2 w3 = cmul(w2, w1);
  v[2] = cmul(v[2], w2);
  v[3] = cmul(v[3], w3);
  if constexpr (R == 4) return;
  const float2 w4 = ld(4);
  v[4] = cmul(v[4], w4);
  v[5] = cmul(v[5], cmul(w4, w1));
  v[6] = cmul(v[6], cmul(w4, w2));
  v[7] = cmul(v[7], cmul(w4, w3));
  if constexpr (R == 8) return;
  const float2 w8 = ld(8);
  const float2 w12 = cmul(w8, w4);
  v[8] = cmul(v[8], w8);
  v[9] = cmul(v[9], cmul(w8, w1));
  v[10] = cmul(v[10], cmul(w8, w2));
  v[11] = cmul(v[11], cmul(w8, w3));
  v[12] = cmul(v[12], w12);
  v[13] = cmul(v[13], cmul(w12, w1));
  v[14] = cmul(v[14], cmul(w12, w2));
  v[15] = cmul(v[15], cmul(w12, w3));
  if constexpr (R == 16) return;
  const float2 w16 = ld(16);
  const float2 w20 = cmul(w16, w4), w24 = cmul(w16, w8), w28 = cmul(w24, w4);
  const float2 wb[4] = {w16, w20, w24, w28};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    v[16 + 4 * q] = cmul(v[16 + 4 * q], wb[q]);
    v[17 + 4 * q] = cmul(v[17 + 4 * q], cmul(wb[q], w1));
    v[18 + 4 * q] = cmul(v[18 + 4 * q], cmul(wb[q], w2));
    v[19 + 4 * q] = cmul(v[19 + 4 * q], cmul(wb[q], w3));
  }
}

// Shape of the transform: T threads, P = N/T points each. SH = (PL << 4) | REV.
// With PL = 0 the passes have radix min(32, P) and the pass that takes what is
// left (REM bits) comes last, or first when REV (a transform whose first pass
// must match the previous transform's last one: the inverse of a convolution
// that keeps the forward's order). Otherwise PL lists the passes' radix bits,
// one hex digit each, the first pass in the lowest digit, taken in reverse order
// when REV (so the inverse again starts with the forward's last radix).
template <int N, int T, int SH = 0>
struct FftShape {
  static constexpr int LOGN = clog2(N);
  static constexpr int P = N / T;
  static constexpr int RBMAX = cmin(5, clog2(P));
  static constexpr int REM = LOGN % RBMAX;
  static constexpr int PL = SH >> 4;
  static constexpr bool REV = (SH & 1) != 0;
  static constexpr int ndig(int p) { return p ? 1 + ndig(p >> 4) : 0; }
  static constexpr int ND = ndig(PL);
  static constexpr int digit(int k) { return REV ? (PL >> (4 * (ND - 1 - k))) & 15 : (PL >> (4 * k)) & 15; }
  static constexpr int plan_rb(int done, int k = 0) { return done == 0 ? digit(k) : plan_rb(done - digit(k), k + 1); }
  static constexpr int plan_sum(int k = 0) { return k == ND ? 0 : digit(k) + plan_sum(k + 1); }
  static constexpr bool plan_ok(int k = 0) { return k == ND ? true : (digit(k) >= 1 && digit(k) <= clog2(P) && plan_ok(k + 1)); }
  static_assert(PL == 0 || (plan_sum() == LOGN && plan_ok()), "pass plan must cover log2 N with radices <= P");
  static constexpr int rb(int done) {
    return PL ? plan_rb(done) : (REV && REM != 0 && done == 0) ? REM : cmin(RBMAX, LOGN - done);
  }
  static constexpr bool last(int done) { return done + rb(done) >= LOGN; }
};

// Twiddles and R-point DFTs of one pass on the P points a thread holds
// (butterfly k in v[k*R .. k*R+R), butterfly index j = tid + k*T).
template <int N, int T, bool INV, int DONE, int SH = 0>
__device__ __forceinline__ void pass_compute(float2* v, int tid) {
  using S = FftShape<N, T, SH>;
  constexpr int R = 1 << S::rb(DONE);
  constexpr int Ns = 1 << DONE;
#pragma unroll
  for (int k = 0; k < S::P / R; ++k) {
    if constexpr (Ns > 1) {
      const int j = tid + k * T;
      const int kk = j & (Ns - 1);
      apply_twiddles<R, Ns * R, INV>(v + k * R, kk);
    }
    dft_reg<R, INV>(v + k * R);
  }
}

// Stockham load of one pass: value r of butterfly j sits at j + r*N/R.
template <int N, int T, int DONE, int SH = 0>
__device__ __forceinline__ void pass_load(const float2* sm, float2* v, int tid) {
  using S = FftShape<N, T, SH>;
  constexpr int R = 1 << S::rb(DONE);
#pragma unroll
  for (int k = 0; k < S::P / R; ++k) {
#pragma unroll
    for (int r = 0; r < R; ++r) v[k * R + r] = sm[fft_pad<N, T>(tid + k * T + r * (N / R))];
  }
}

// Stockham store of one pass: output r of butterfly j goes to (j - kk)*R + kk + r*Ns.
template <int N, int T, int DONE, int SH = 0>
__device__ __forceinline__ void pass_store(float2* sm, const float2* v, int tid) {
  using S = FftShape<N, T, SH>;
  constexpr int R = 1 << S::rb(DONE);
  constexpr int Ns = 1 << DONE;
#pragma unroll
  for (int k = 0; k < S::P / R; ++k) {
    const int j = tid + k * T;
    const int kk = j & (Ns - 1);
    const int e = (j - kk) * R + kk;
#pragma unroll
    for (int r = 0; r < R; ++r) sm[fft_pad<N, T>(e + r * Ns)] = v[k * R + r];
  }
}

// Passes DONE.. that go shared memory -> shared memory, stopping before the
// last pass when STOP_BEFORE_LAST (the caller finishes it with its own store).
template <int N, int T, bool INV, int DONE, bool STOP_BEFORE_LAST, int SH = 0, class Sync>
__device__ __forceinline__ void smem_passes(float2* sm, int tid, Sync sync) {
  using S = FftShape<N, T, SH>;
  if constexpr (DONE < S::LOGN) {
    if constexpr (!(STOP_BEFORE_LAST && S::last(DONE))) {
      float2 v[S::P];
      pass_load<N, T, DONE, SH>(sm, v, tid);
      pass_compute<N, T, INV, DONE, SH>(v, tid);
      sync();
      pass_store<N, T, DONE, SH>(sm, v, tid);
      sync();
      smem_passes<N, T, INV, DONE + S::rb(DONE), STOP_BEFORE_LAST, SH>(sm, tid, sync);
    }
  }
}

// Start of the last pass.
template <int N, int T, int DONE = 0, int SH = 0>
constexpr int last_pass_done() {
  using S = FftShape<N, T, SH>;
  if constexpr (S::last(DONE)) return DONE;
  else return last_pass_done<N, T, DONE + S::rb(DONE), SH>();
}

// In-place transform of sm[fft_pad<N, T>(0..N)) by the T threads with tid in [0, T).
// Callers synchronise before (data written) and may read results right after.
template <int N, int T, bool INV, class Sync>
__device__ __forceinline__ void fft_smem(float2* sm, int tid, Sync sync) {
  static_assert((N & (N - 1)) == 0 && N >= 2 * T, "bad FFT shape");
  smem_passes<N, T, INV, 0, false>(sm, tid, sync);
}

// Threads per transform: 16 or 32 points per thread, whichever measured faster
// on B200 for the size (an 18 x 3456-row batch at every side): 32 points where
// radix-32 passes save a pass (512, 1024, 16384) or tie it (4096), 16 elsewhere
// (half the registers per thread, so twice the resident warps).
__host__ __device__ constexpr int fft_points_per_thread(int n) {
  return (n == 512 || n == 1024 || n == 4096 || n == 16384) ? 32 : 16;
}
__host__ __device__ constexpr int fft_threads(int n) { return n / fft_points_per_thread(n); }
// Threads per CTA: whole warps; small transforms share a warp.
__host__ __device__ constexpr int fft_cta_threads(int n) { return fft_threads(n) >= 128 ? fft_threads(n) : 128; }
// Transforms per CTA.
__host__ __device__ constexpr int fft_per_cta(int n) { return fft_cta_threads(n) / fft_threads(n); }

}  // namespace fi
