// Internal declarations shared by the C-ABI layer and the kernels.
//
// Device memory layout (all fp32):
//   state   [M+1][S][L]   slot array per layer l = 0..M, S = B*D streams with
//                          stream index s = d*B + b (a channel's sequences are
//                          adjacent). For a position t below the current one,
//                          slot (l, s, t) holds the activation a^l_t; at or
//                          above it, slot (l, s, t) holds layer l's accumulator
//                          (page, "Ottimizzazione della Memoria": b^l_i is kept
//                          in a^l_i's place). l = 0 holds the tokens.
//   taps    [M][D][L]     filters widened to fp32 (bf16 values are exact in fp32).
//   spectra per level q with U = 2^q >= fft_from: [M][D][U+1] complex, the
//                          real-input DFT of h[0..2U) divided by 2U.
//   twiddle [2^15]         exp(-2 pi i m / 2^15), computed in double on the host.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <string>

#include "../../include/fi.h"

namespace fi {

constexpr int kTwiddleLog2 = 15;              // table covers real FFTs of length <= 2^15
constexpr int kTwiddleN = 1 << kTwiddleLog2;
constexpr int kMaxFftLog2 = 14;               // complex FFT points held in one CTA's shared memory
constexpr int kMinFftLog2 = 6;

enum KernelClass { KC_CHUNK = 0, KC_DIRECT = 1, KC_FFT = 2, KC_TOKEN = 3, KC_LAZY = 4, KC_TC = 5 };

struct Dims {
  int M, D, L, B, S;   // layers, channels, max length, batch, streams
  int P;               // log2 L
  int bf16;            // tokens and filters are bf16
};

__host__ __device__ inline size_t slot_index(const Dims& g, int l, int s, int t) {
  return ((size_t)l * g.S + s) * (size_t)g.L + t;
}

__device__ __forceinline__ float round_act(float v, int bf16) {
  return bf16 ? __bfloat162float(__float2bfloat16_rn(v)) : v;
}

__device__ __forceinline__ float load_token(const void* p, size_t i, int bf16) {
  return bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i])
              : reinterpret_cast<const float*>(p)[i];
}

inline int ilog2(uint32_t v) { int r = 0; while ((1u << (r + 1)) <= v && r < 31) ++r; return r; }
inline bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }
inline int lowbit(int i) { return i & -i; }
inline int highbit(int i) { int r = 1; while ((int64_t)r * 2 <= i) r *= 2; return r; }

// Programmatic dependent launch. Block kernels call pdl_launch_dependents() on
// entry, so that the next launch on the stream, the chunk kernel (launched with
// programmatic stream serialization), may start once every block CTA is
// running; the chunk kernel loads what no block writes (taps, noise) and then
// calls pdl_wait_primary(), which returns when the preceding grid has completed
// and its writes are visible. Both are no-ops for a launch without the attribute.
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait_primary() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// ---------------------------------------------------------------- launchers (kernels/*.cu)
// All return cudaSuccess or the launch error.

// Red cells + blocks of one position for all streams (fi_step, lazy). block_u > 0
// (1, 2, 4 or kTokenBlockMax) also adds the direct block of step t (side
// block_u = lowbit(t)) in the same launch, before the red cells; it needs
// M <= kTokenMaxLayers (token_block_fused says whether a shape qualifies).
constexpr int kTokenBlockMax = 8;
constexpr int kTokenMaxLayers = 32;
inline bool token_block_fused(const Dims& g, int U) { return g.M <= kTokenMaxLayers && U >= 1 && U <= kTokenBlockMax; }
cudaError_t launch_token(const Dims& g, float* state, const float* taps, int t, const void* x_t,
                         const float* eps_t, float eps_scale, float* y_t, cudaStream_t st, int block_u = 0);

// Direct block of step i (side U = lowbit(i)) from HBM for all layers and streams;
// overwrite = the block is the first to reach its targets (i a power of two).
// Block launchers take t_min: targets below it are not written (t_min <= i: all).
cudaError_t launch_tile_direct(const Dims& g, float* state, const float* taps, int i,
                               int t_min, cudaStream_t st);

// FFT block of step i (side U = lowbit(i), 2^kMinFftLog2 <= U <= 2^kMaxFftLog2).
// pdl: launched with programmatic stream serialization (worth it after a chunk
// kernel that fills nearly every SM; with many idle SMs the early grid would
// settle there and run on fewer SMs).
cudaError_t launch_tile_fft(const Dims& g, float* state, const float2* spectrum_q,
                            const float2* twiddle, int i, int t_min, cudaStream_t st, bool pdl = false);

// Spectra of one level q for all (layer, channel).
cudaError_t launch_spectra(const Dims& g, const float* taps, float2* spectrum_q,
                           const float2* twiddle, int q, cudaStream_t st);

// Blocks of side U = m * 2^kMaxFftLog2 (m >= 2): segment spectra of one level,
// gspec[M][D][2m-1][N+1] (segment e = rFFT_2N(h[eN .. eN+2N)) / 2N), and the
// block itself (forward transforms into xs[M*S][m][N+1], then inverse ones).
cudaError_t launch_part_spectra(const Dims& g, const float* taps, float2* gspec, const float2* twiddle, int m,
                                cudaStream_t st);
cudaError_t launch_part_block(const Dims& g, float* state, float2* xs, const float2* gspec, const float2* twiddle,
                              int i, int t_min, cudaStream_t st);

// Tensor-core block of side U (k_tile_tc.cu): M-tile rows MT (64 or 128), J
// target tiles per product, NR operand rows (B*J padded), K steps of 16 over
// U + (J-1)*MT reversed sources, accumulator columns, split (fp32 contexts:
// three bf16 products), dynamic shared memory and grid.
struct TcPlan {
  int U, MT, J, NR, K, tmem_cols, split, grid, ipc, per_sm;   // ipc: items per pass of a CTA
  size_t smem, item_bytes;
};
cudaError_t tc_prepare(const Dims& g, int U, int split, int num_sms, TcPlan* out);
cudaError_t launch_tile_tc(const Dims& g, float* state, const float* taps, const TcPlan& p, int i, int* err,
                           int wait_limit, cudaStream_t st);

// Which on-chip block pieces run at which step of a chunk (built on the host):
// entries sorted by step, e[first[r] .. first[r+1]) run at step r; entry =
// step | s_lo << 7 | t_lo << 14 | kind << 21 (sources [s_lo, s_lo+ns) to
// targets [t_lo, t_lo+nd), positions relative to the chunk start).
constexpr int kChunkMaxSteps = 64;
constexpr int kChainLags = 2;   // re-timed chunks: lags the chain adds itself (pieces take the rest)
constexpr int kChunkMaxEntries = 192;
struct ChunkTable {
  int n;
  int lag1;      // lags 1..lag1 are added by the chain itself (0 or kChainLags); pieces cover the rest
  uint16_t first[kChunkMaxSteps + 1];
  uint32_t e[kChunkMaxEntries];
};
// retimed = the whole chunk runs in one launch: the chain takes the terms of
// lags 1..kChainLags, the page's tiling of the remaining pairs runs kChainLags
// positions ahead (its targets shifted by kChainLags), with blocks of side 8 and
// up cut into pieces spread over steps; else the page's blocks, one per step.
// coarse: the 16-source halves of the side-32 blocks stay 16 x 16 pieces
// (fewer pieces; measured faster when the chain is short, M <= kCoarseMaxLayers).
constexpr int kCoarseMaxLayers = 8;
bool build_chunk_table(int chunk, bool retimed, ChunkTable* tab, bool coarse = false);
// Sources and targets of a piece kind (for the table's test hook).
int chunk_piece_sources(int kind);
int chunk_piece_targets(int kind);

// The chunk kernel: positions [p0, p1) inside the aligned chunk [c, c+chunk),
// small blocks (side < chunk) on chip, red cells, blocks and the sampler.
struct ChunkArgs {
  float* state;
  const float* taps;
  const void* x0;        // token at p0 when first_call (dtype of the context), else NULL
  const float* eps;      // [n][B][D] relative to gen_base
  float eps_scale;
  float* y_out;          // [n][B][D] relative to gen_base
  float* rec;            // NULL or [M][n][B][D]
  int n_gen;             // n of the generate call (rec stride)
  int gen_base;          // first position of the generate call
  int c, chunk, p0, p1;  // chunk start, chunk length, positions to produce
  int last_done;         // last step whose blocks have reached HBM before this launch
  int* err;              // device flag set to 1 when a bounded wait gives up
  int wait_limit;        // barrier checks before a wait gives up
  int trigger;           // let the next block launch (programmatic) start early
  ChunkTable tab;        // filled by launch_chunk
};

// Default number of barrier checks before a device-side wait gives up (each
// check lasts at most about a microsecond, so this is far beyond any real wait).
constexpr int kDefaultWaitLimit = 1 << 20;
cudaError_t launch_chunk(const Dims& g, const ChunkArgs& a, int streams_per_cta, cudaStream_t st);
cudaError_t configure_chunk(size_t smem);   // allow `smem` bytes of dynamic shared memory
int chunk_streams_per_cta(const Dims& g, int chunk, int num_sms, size_t max_smem);
// A chunk CTA of this shape takes a whole SM (every register), so no other
// grid's CTA can share its SM while it runs.
bool chunk_cta_fills_sm(const Dims& g, int streams_per_cta);
size_t chunk_smem_bytes(const Dims& g, int chunk, int streams_per_cta);

// Lazy sums of position t for all layers: slot(l, s, t) = sum_{s' < t} h^l[t-s'] a^{l-1}_{s'}.
cudaError_t launch_lazy_sums(const Dims& g, float* state, const float* taps, int t, cudaStream_t st);

// Prompt prefill: tokens x[p][B][D] into layer 0, then for every layer the
// offline causal convolution of the prompt (FFT of 2N points, N = 2^q >= p with
// q = prefix_transform_log2(p) <= kMaxFftLog2) and the block; spec is scratch
// for M*D*(N+1) complex values. y_out [p][B][D] (layer M) and rec [M][p][B][D]
// may be NULL.
int prefix_transform_log2(int p);
cudaError_t launch_prefix(const Dims& g, float* state, const float* taps, float2* spec, const float2* twiddle, int p,
                          const void* x, float* y_out, float* rec, cudaStream_t st);

// Debug: batch of complex FFTs with the tile FFT code.
cudaError_t launch_debug_fft(int log2n, int count, const float2* in, float2* out, int inverse,
                             const float2* twiddle, cudaStream_t st);

// Channel-mixing block (MLP + GELU) state: weights copied from the caller, the
// hidden activations and red cells of one position, and the position record a
// captured position reads.
constexpr int kMlpGroup = 8;      // sequences one CTA applies each weight row to
constexpr int kMlpBlockMax = 8;   // blocks of side <= this run in the position's own launches
// One position of the block: t, and where its outputs go (y^l_t to
// rec [M][n_gen][B][D] and, l = M, y_out [n_gen][B][D], rows t - gen_base; eps
// [n_gen][B][D] noise of the sampler, NULL: no next token is written).
struct MlpPos {
  int t, gen_base, n_gen;
  float eps_scale;
  const float* eps;
  float* y_out;
  float* rec;
};
struct MlpBlock {
  int hidden = 0;            // Dh; 0 = the elementwise tanh block
  float* w1 = nullptr;       // [M][Dh][D]
  float* b1 = nullptr;       // [M][Dh]
  float* w2 = nullptr;       // [M][D][Dh]
  float* b2 = nullptr;       // [M][D]
  float* z = nullptr;        // [B][Dh] scratch
  float* y = nullptr;        // [B][D] scratch: the next layer's red cells
  MlpPos* pos = nullptr;     // the position a captured position reads (advanced by the capture)
};
// Dynamic shared memory the block's kernels need (must fit one CTA).
size_t mlp_smem_bytes(const Dims& g, int hidden);
// Token x [B][D] into layer 0 at position t.
cudaError_t launch_mlp_token(const Dims& g, float* state, const void* x, int t, cudaStream_t st);
// Shared-memory limits of the block's kernels (call before launching or capturing).
cudaError_t prepare_mlp(const Dims& g, const MlpBlock& m);
// Layer l at position p.t (or at *p_dev, when p_dev is given: a captured
// position): the block's two products for every (sequence, channel). The
// block's output goes to the state (l < M) or, with noise, to the next token.
// The block of step t must have run before layer 1.
cudaError_t launch_mlp_layer(const Dims& g, float* state, const float* taps, const MlpBlock& m, int l,
                             const MlpPos& p, const MlpPos* p_dev, cudaStream_t st);
// The small block of step p.t (or *p_dev's), side lowbit(t) <= kMlpBlockMax,
// for every layer and stream (nothing for t = 0 or a wider block, run from HBM
// before), then layer 1's red cells into m.y and the records. Launched before
// layer 1's launches.
cudaError_t launch_mlp_block(const Dims& g, float* state, const float* taps, const MlpPos& p, const MlpPos* p_dev,
                             float* ybuf, cudaStream_t st);
// p_dev->t += 1 (the last node of a captured position); *p_dev = v.
cudaError_t launch_mlp_next(MlpPos* p_dev, cudaStream_t st);
cudaError_t launch_mlp_set(MlpPos* p_dev, const MlpPos& v, cudaStream_t st);

// Message returned by fi_last_error() for the calling thread.
void set_last_error(const std::string& msg);

// Conversions for fi_init / fi_read_activations.
cudaError_t launch_widen_filters(const void* h, int bf16, size_t n, float* out, cudaStream_t st);
cudaError_t launch_read_layer(const Dims& g, const float* state, int layer, int pos, float* dst,
                              cudaStream_t st);

}  // namespace fi
