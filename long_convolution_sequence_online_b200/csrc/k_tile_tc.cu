// Gray blocks on the 5th-generation tensor cores (tcgen05, accumulators in
// tensor memory).
//
// The block of step i (side U = lowbit(i), the page's tau(a, [i-U, i-1], h,
// [i, i+U-1]), "Definizione di Aggregazione di Contribuzione") is, for one
// (layer, channel) and the B sequences that share its filter, a Toeplitz
// product Y[u'][b] = sum_u h[U + u' - u] X[u][b]. Written with the sources in
// reverse order, kappa = i - 1 - u, the matrix becomes a Hankel one,
// A[r][kappa] = h[r + kappa + 1], whose rows are overlapping windows of the
// filter. The tensor-core operand descriptor can express that directly: a table
// of 16-byte entries, entry sigma = h[sigma+1 .. sigma+8] in bf16, read as a
// K-major operand with both the row-group stride and the K-half stride equal to
// one core matrix (128 bytes, 8 entries). Nothing of the U x U matrix is ever
// materialised: the table holds 2U entries.
//
// Several target tiles share one product: tile j (targets i + j*MT .. + MT) uses
// the same table when its sources sit kappa = j*MT further along, so the B
// operand holds, for each tile j of a group and each sequence b, one row with
// the sources placed at kappa in [j*MT, j*MT + U) and zeros elsewhere. Narrow
// batches (B = 4) thus still fill N = B*J >= 8 columns of the instruction.
//
// Precision: bf16 contexts hold bf16-exact filters and activations, so one
// bf16 x bf16 -> fp32 product per K step is exact up to fp32 accumulation. fp32
// contexts split both operands, v = hi + lo with hi = bf16(v) and
// lo = bf16(v - hi), and add the three products hi*hi + hi*lo + lo*hi (the
// dropped lo*lo term and the residuals are below 2^-16 relative per product).
//
// A CTA works through passes of one or more (layer, channel) items: operand
// builder warps write the tables and B operands of a pass into shared memory,
// one thread issues the MMAs of every item and group (each into its own
// accumulator columns) and commits them to an mbarrier, and drain warps read
// their 32 accumulator lanes and add them to the targets in HBM; two stages
// let the three roles work on consecutive passes at once (details at the
// kernel). Every wait is bounded.
#include "fi_internal.cuh"

namespace fi {

namespace {

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// K-major operand without swizzle: start, leading (K-half) and stride
// (8-row group) byte offsets, all in 16-byte units; version 1 (bits 46-47).
__device__ __forceinline__ uint64_t smem_desc(uint32_t start, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((start >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}

// Instruction descriptor, kind::f16: fp32 accumulator, bf16 A and B, both
// K-major, N >> 3 at bit 17, M >> 4 at bit 24.
__host__ __device__ constexpr uint32_t tc_idesc(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

__device__ __forceinline__ void mma_bf16(uint32_t dtmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(dtmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_addr(bar)) : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ bool bar_try(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok) : "r"(smem_addr(bar)), "r"(parity), "r"(1000u) : "memory");
  return ok != 0;
}

__device__ __forceinline__ bool bar_wait(uint64_t* bar, uint32_t parity, int limit) {
  for (int it = 0; it < limit; ++it)
    if (bar_try(bar, parity)) return true;
  return false;
}

// 8 accumulator columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int k = 0; k < 8; ++k) v[k] = __uint_as_float(r[k]);
}

// 16 accumulator columns of this warp's 32 lanes.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
  for (int k = 0; k < 16; ++k) v[k] = __uint_as_float(r[k]);
}

__device__ __forceinline__ uint16_t bf16_bits(float v) {
  return __bfloat16_as_ushort(__float2bfloat16_rn(v));
}
// hi = bf16(v), lo = bf16(v - hi)
__device__ __forceinline__ void split_bf16(float v, uint16_t& hi, uint16_t& lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(v);
  hi = __bfloat16_as_ushort(h);
  lo = bf16_bits(v - __bfloat162float(h));
}

}  // namespace

// Byte offset of element (row n, column k) of a K-major operand with R rows
// (R a multiple of 8) in core-matrix order: core (n/8, k/8) at
// ((k/8)*(R/8) + n/8) * 128, rows 16 bytes apart, elements 2 bytes apart.
__host__ __device__ constexpr uint32_t tc_b_offset(int R, int n, int k) {
  return (uint32_t)(((k >> 3) * (R >> 3) + (n >> 3)) * 128 + (n & 7) * 16 + (k & 7) * 2);
}

// Warp roles: warps 0-3 build operands, warp 4 issues the MMAs, warps 5-8 drain
// the accumulators (warp w reads tensor-memory lanes 32*(w % 4) .. +31). Two
// stages of operands and accumulators let pass p+1 load while pass p multiplies
// and pass p-1 drains. Per stage s, three mbarriers: full (loaders -> MMA),
// done (MMA commit -> loaders, which may overwrite the operands, and -> drain),
// empty (drain -> MMA, which may overwrite the accumulators). Use k of a stage
// waits on parity k & 1; no barrier runs more than one phase ahead of a waiter.
constexpr int kTcLoadWarps = 4;
constexpr int kTcMmaWarp = kTcLoadWarps;
constexpr int kTcDrainWarp0 = kTcLoadWarps + 1;
constexpr int kTcThreads = 32 * (kTcLoadWarps + 1 + 4);

__device__ __forceinline__ void bar_arrive(uint64_t* bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_addr(bar)) : "memory");
}
// OR of `v` over the operand-builder warps (named barrier 1), so they leave
// their loop together.
__device__ __forceinline__ bool loaders_any(bool v) {
  uint32_t out;
  asm volatile("{\n\t.reg .pred q, p;\n\tsetp.ne.u32 q, %1, 0;\n\tbar.red.or.pred p, 1, %2, q;\n\tselp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(out) : "r"((uint32_t)v), "r"(32 * kTcLoadWarps) : "memory");
  return out != 0;
}
// Bounded wait that also gives up once another role has given up.
__device__ __forceinline__ bool bar_wait_or_abort(uint64_t* bar, uint32_t parity, int limit, volatile int* abort_flag) {
  for (int it = 0; it < limit; ++it) {
    if (bar_try(bar, parity)) return true;
    if (*abort_flag) return false;
  }
  return false;
}

template <int MT, bool SPLIT>
__global__ void __launch_bounds__(kTcThreads) k_tile_tc(Dims g, float* __restrict__ state, const float* __restrict__ taps,
                                                        TcPlan p, int i, int overwrite, int* err, int wait_limit) {
  pdl_launch_dependents();
  extern __shared__ __align__(1024) unsigned char tsm[];
  __shared__ uint64_t full_bar[2], done_bar[2], empty_bar[2];
  __shared__ uint32_t tmem_base_s;
  __shared__ int abort_s;
  __shared__ int col_ofs[512];   // accumulator column -> target offset from the item's row base, or -1
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int U = p.U, J = p.J, NR = p.NR, K = p.K, IPC = p.ipc;
  const int NT = U / MT, groups = NT / J;
  const int cols = groups * NR;                 // accumulator columns of one item
  const uint32_t idesc = tc_idesc(MT, NR);
  const size_t xbytes = (size_t)NR * K * 2;
  const size_t stage_bytes = (size_t)IPC * p.item_bytes;
  // Item k of stage s, at tsm + s * stage_bytes + k * item_bytes: table hi
  // [2U][16 B], (table lo), X hi [NR rows][K], (X lo).
  auto item_base = [&](int st, int k) { return tsm + (size_t)st * stage_bytes + (size_t)k * p.item_bytes; };
  auto tab_hi = [&](int st, int k) { return item_base(st, k); };
  auto tab_lo = [&](int st, int k) { return item_base(st, k) + (size_t)32 * U; };
  auto x_hi = [&](int st, int k) { return item_base(st, k) + (SPLIT ? 2 : 1) * (size_t)32 * U; };
  auto x_lo = [&](int st, int k) { return x_hi(st, k) + xbytes; };

  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_addr(&tmem_base_s)), "r"(p.tmem_cols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  // Column c of an item: group gi = c / NR, operand row n = c % NR = j*B + b;
  // its target for accumulator row r is slot (l, d*B + b, i + (gi*J + j)*MT + r),
  // i.e. the item's row base plus b*L + (gi*J + j)*MT.
  for (int c = tid; c < cols; c += blockDim.x) {
    const int gi = c / NR, n = c - gi * NR;
    const int j = n / g.B, b = n - j * g.B;
    col_ofs[c] = n < J * g.B ? b * g.L + (gi * J + j) * MT : -1;
  }
  if (tid == 0) {
    for (int st = 0; st < 2; ++st) {
      asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(&full_bar[st])), "r"(32 * kTcLoadWarps) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(smem_addr(&done_bar[st])) : "memory");
      asm volatile("mbarrier.init.shared::cta.b64 [%0], 128;" ::"r"(smem_addr(&empty_bar[st])) : "memory");
    }
    abort_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  const uint32_t tmem = tmem_base_s;
  volatile int* abort_flag = &abort_s;
  auto give_up = [&]() {
    *abort_flag = 1;
    atomicExch(err, 1);
  };

  const long items = (long)g.M * g.D;
  const long first = (long)blockIdx.x * IPC, stride = (long)gridDim.x * IPC;
  const int npass = first < items ? (int)((items - 1 - first) / stride) + 1 : 0;
  int last_commit = -1;                          // MMA issuer: last pass committed

  if (warp < kTcLoadWarps) {
    // ------------------------------------------------------------ operand builders
    const int lt = tid;                          // 0..127
    for (int ps = 0; ps < npass; ++ps) {
      const int st = ps & 1;
      const long base = first + (long)ps * stride;
      const int nk = (int)(items - base < IPC ? items - base : IPC);
      const bool free = ps < 2 || bar_wait_or_abort(&done_bar[st], ((ps - 2) >> 1) & 1, wait_limit, abort_flag);
      if (loaders_any(!free)) {
        if (lt == 0) give_up();
        break;
      }
      // Tables: entry s = h[s+1 .. s+8] (taps beyond 2U-1 meet only zero
      // sources), and the B operands zeroed.
      for (int k = 0; k < nk; ++k) {
        const float* hp = taps + (size_t)(base + k) * g.L;       // item = (l-1)*D + d
        // entries 8t .. 8t+7 from taps h[8t .. 8t+15] (four 16-byte loads)
        for (int t8 = lt; t8 < 2 * U / 8; t8 += 32 * kTcLoadWarps) {
          float hv[16];
#pragma unroll
          for (int f = 0; f < 4; ++f) {
            const int o = 8 * t8 + 4 * f;
            const float4 v = o + 4 <= g.L ? __ldg(reinterpret_cast<const float4*>(hp + o)) : make_float4(0.f, 0.f, 0.f, 0.f);
            hv[4 * f] = v.x; hv[4 * f + 1] = v.y; hv[4 * f + 2] = v.z; hv[4 * f + 3] = v.w;
          }
#pragma unroll
          for (int m = 0; m < 8; ++m) {
            uint32_t wh[4], wl[4];
#pragma unroll
            for (int e = 0; e < 8; e += 2) {
              const float v0 = hv[m + 1 + e], v1 = hv[m + 2 + e];
              uint16_t h0, l0, h1, l1;
              if constexpr (SPLIT) {
                split_bf16(v0, h0, l0);
                split_bf16(v1, h1, l1);
              } else {
                h0 = bf16_bits(v0); h1 = bf16_bits(v1); l0 = l1 = 0;
              }
              wh[e / 2] = (uint32_t)h0 | ((uint32_t)h1 << 16);
              wl[e / 2] = (uint32_t)l0 | ((uint32_t)l1 << 16);
            }
            const size_t eo = (size_t)(8 * t8 + m) * 16;
            *reinterpret_cast<uint4*>(tab_hi(st, k) + eo) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
            if constexpr (SPLIT) *reinterpret_cast<uint4*>(tab_lo(st, k) + eo) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
          }
        }
        for (size_t q = (size_t)lt * 16; q < xbytes; q += 128 * 16) {
          *reinterpret_cast<uint4*>(x_hi(st, k) + q) = make_uint4(0, 0, 0, 0);
          if constexpr (SPLIT) *reinterpret_cast<uint4*>(x_lo(st, k) + q) = make_uint4(0, 0, 0, 0);
        }
      }
      asm volatile("bar.sync 1, %0;" ::"r"(32 * kTcLoadWarps) : "memory");
      // B operands: the sources of each (tile j, sequence b) row. A thread takes
      // 8 consecutive sources of one sequence (one 32-byte sector) and writes
      // them as one 16-byte core-matrix row; consecutive threads take
      // consecutive sequences, so a warp's stores fill whole core matrices.
      // Several tasks per round: all their global loads go out before the first
      // conversion waits on data, so a thread keeps up to eight loads in flight.
      const int oct = U / 8;
      const int ntask = nk * g.B * oct;
      constexpr int kTasks = SPLIT ? 2 : 4;   // split operands need twice the registers per task
      for (int w0 = lt; w0 < ntask; w0 += kTasks * 128) {
        float4 v0[kTasks], v1[kTasks];
#pragma unroll
        for (int u = 0; u < kTasks; ++u) {
          const int w = w0 + u * 128;
          if (w < ntask) {
            const int k = w / (g.B * oct), wr = w - k * (g.B * oct);
            const int q8 = wr / g.B, b = wr - q8 * g.B;
            const long item = base + k;
            const int l = (int)(item / g.D) + 1, d = (int)(item - (long)(l - 1) * g.D);
            const float4* src = reinterpret_cast<const float4*>(state + slot_index(g, l - 1, d * g.B + b, i - U) + 8 * q8);
            v0[u] = src[0];
            v1[u] = src[1];
          }
        }
#pragma unroll
        for (int u = 0; u < kTasks; ++u) {
          const int w = w0 + u * 128;
          if (w >= ntask) break;
          const int k = w / (g.B * oct), wr = w - k * (g.B * oct);
          const int q8 = wr / g.B, b = wr - q8 * g.B;
          // source 8 q8 + e sits at kappa = U - 1 - 8 q8 - e: kappa kb + m holds element 7 - m
          const int kb = U - 8 - 8 * q8;
          const float vv[8] = {v1[u].w, v1[u].z, v1[u].y, v1[u].x, v0[u].w, v0[u].z, v0[u].y, v0[u].x};
          uint32_t wh[4], wl[4];
#pragma unroll
          for (int m = 0; m < 8; m += 2) {
            uint16_t h0, l0, h1, l1;
            if constexpr (SPLIT) {
              split_bf16(vv[m], h0, l0);
              split_bf16(vv[m + 1], h1, l1);
            } else {
              h0 = bf16_bits(vv[m]); h1 = bf16_bits(vv[m + 1]); l0 = l1 = 0;
            }
            wh[m / 2] = (uint32_t)h0 | ((uint32_t)h1 << 16);
            wl[m / 2] = (uint32_t)l0 | ((uint32_t)l1 << 16);
          }
          for (int j = 0; j < J; ++j) {
            const uint32_t off = tc_b_offset(NR, j * g.B + b, j * MT + kb);
            *reinterpret_cast<uint4*>(x_hi(st, k) + off) = make_uint4(wh[0], wh[1], wh[2], wh[3]);
            if constexpr (SPLIT) *reinterpret_cast<uint4*>(x_lo(st, k) + off) = make_uint4(wl[0], wl[1], wl[2], wl[3]);
          }
        }
      }
      fence_proxy_async();   // generic-proxy writes -> visible to the tensor core
      bar_arrive(&full_bar[st]);
    }
  } else if (warp == kTcMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t lbo_b = (uint32_t)(NR / 8) * 128;
      for (int ps = 0; ps < npass; ++ps) {
        const int st = ps & 1;
        const long base = first + (long)ps * stride;
        const int nk = (int)(items - base < IPC ? items - base : IPC);
        if (!bar_wait_or_abort(&full_bar[st], (ps >> 1) & 1, wait_limit, abort_flag) ||
            (ps >= 2 && !bar_wait_or_abort(&empty_bar[st], ((ps - 2) >> 1) & 1, wait_limit, abort_flag))) {
          give_up();
          break;
        }
        fence_after_sync();
        for (int k = 0; k < nk; ++k) {
          const uint32_t th = smem_addr(tab_hi(st, k)), tl = smem_addr(tab_lo(st, k));
          const uint32_t xh = smem_addr(x_hi(st, k)), xl = smem_addr(x_lo(st, k));
          for (int gi = 0; gi < groups; ++gi) {
            const uint32_t dcol = tmem + (uint32_t)((st * IPC + k) * cols + gi * NR);
            for (int ks = 0; ks < K / 16; ++ks) {
              const uint32_t a_off = (uint32_t)(gi * J * MT + 16 * ks) * 16;
              const uint32_t b_off = (uint32_t)(2 * ks) * lbo_b;
              const uint64_t ah = smem_desc(th + a_off, 128, 128);
              const uint64_t bh = smem_desc(xh + b_off, lbo_b, 128);
              mma_bf16(dcol, ah, bh, idesc, ks > 0 ? 1u : 0u);
              if constexpr (SPLIT) {
                const uint64_t al = smem_desc(tl + a_off, 128, 128);
                const uint64_t bl = smem_desc(xl + b_off, lbo_b, 128);
                mma_bf16(dcol, ah, bl, idesc, 1u);
                mma_bf16(dcol, al, bh, idesc, 1u);
              }
            }
          }
        }
        mma_commit(&done_bar[st]);
        last_commit = ps;
      }
      // The accumulators are released only after the last commit has arrived
      // (a wait of its own, at least the default length: a caller's short wait
      // limit must not release columns that MMAs still write).
      if (last_commit >= 0)
        bar_wait(&done_bar[last_commit & 1], (last_commit >> 1) & 1, wait_limit > kDefaultWaitLimit ? wait_limit : kDefaultWaitLimit);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ drain
    // Row r of tile (gi*J + j) is target i + (gi*J + j)*MT + r; lane 32q + x of
    // the accumulator (q = warp % 4) holds row 32q + x (MT = 128) or, for
    // MT = 64, rows 16q + x in lanes x < 16 of each quarter.
    const int q = warp & 3;
    const int r = MT == 128 ? 32 * q + lane : 16 * q + lane;
    const bool row_ok = MT == 128 || lane < 16;
    for (int ps = 0; ps < npass; ++ps) {
      const int st = ps & 1;
      const long base = first + (long)ps * stride;
      const int nk = (int)(items - base < IPC ? items - base : IPC);
      // lanes of a warp leave together (the accumulator loads are warp-wide)
      const bool arrived = bar_wait_or_abort(&done_bar[st], (ps >> 1) & 1, wait_limit, abort_flag);
      if (!__all_sync(0xffffffffu, arrived)) {
        if (lane == 0) give_up();
        break;
      }
      fence_after_sync();
      for (int k = 0; k < nk; ++k) {
        const long item = base + k;
        const int l = (int)(item / g.D) + 1, d = (int)(item - (long)(l - 1) * g.D);
        float* rowbase = state + slot_index(g, l, d * g.B, i + r);
        // 16 columns per round: the old accumulator values (independent of the
        // tensor memory) are all requested first, then the two 8-column loads.
        for (int c0 = 0; c0 < cols; c0 += 16) {
          int ofs[16];
          float old[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            ofs[e] = (c0 + e < cols && row_ok) ? col_ofs[c0 + e] : -1;
            old[e] = (ofs[e] >= 0 && !overwrite) ? rowbase[ofs[e]] : 0.f;
          }
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            if (c0 + 8 * h >= cols) break;       // uniform across the warp
            float v[8];
            tmem_ld8(tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)((st * IPC + k) * cols + c0 + 8 * h), v);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if (ofs[8 * h + e] >= 0) rowbase[ofs[8 * h + e]] = old[8 * h + e] + v[e];
          }
        }
      }
      fence_before_sync();
      bar_arrive(&empty_bar[st]);
    }
  }

  fence_before_sync();
  __syncthreads();
  fence_after_sync();
  if (warp == 0)
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(p.tmem_cols) : "memory");
}

// ------------------------------------------------------------------ host side
static int pow2_at_least(int v) { int r = 1; while (r < v) r <<= 1; return r; }

// CTAs of one plan that fit on an SM: threads, registers and shared memory
// counted from the kernel's attributes (the dynamic shared-memory limit of the
// instantiation only ever grows, since several block sides share it).
template <int MT, bool SPLIT>
static cudaError_t tc_occupancy(const TcPlan& p, int device, int* per_sm) {
  auto kern = k_tile_tc<MT, SPLIT>;
  cudaFuncAttributes fa{};
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  if ((size_t)fa.maxDynamicSharedSizeBytes < p.smem)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)p.smem);
  if (e == cudaSuccess)
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout, (int)cudaSharedmemCarveoutMaxShared);
  if (e != cudaSuccess) return e;
  int sm_smem = 0, sm_regs = 0, sm_threads = 0, sm_blocks = 0, reserved = 0;
  if ((e = cudaDeviceGetAttribute(&sm_smem, cudaDevAttrMaxSharedMemoryPerMultiprocessor, device)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&sm_regs, cudaDevAttrMaxRegistersPerMultiprocessor, device)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&sm_threads, cudaDevAttrMaxThreadsPerMultiProcessor, device)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&sm_blocks, cudaDevAttrMaxBlocksPerMultiprocessor, device)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&reserved, cudaDevAttrReservedSharedMemoryPerBlock, device)) != cudaSuccess)
    return e;
  const size_t per_cta_smem = p.smem + fa.sharedSizeBytes + (size_t)reserved;
  const int warps = kTcThreads / 32;
  const int regs_cta = ((fa.numRegs * 32 + 255) / 256 * 256) * warps;   // 256-register allocation units per warp
  int n = sm_threads / kTcThreads;
  if (sm_blocks < n) n = sm_blocks;
  if (regs_cta > 0 && sm_regs / regs_cta < n) n = sm_regs / regs_cta;
  if ((int)(sm_smem / per_cta_smem) < n) n = (int)(sm_smem / per_cta_smem);
  *per_sm = n;
  return cudaSuccess;
}

cudaError_t tc_prepare(const Dims& g, int U, int split, int num_sms, TcPlan* out) {
  if (U < 64 || (U & (U - 1)) || U > g.L / 2) return cudaErrorInvalidValue;
  TcPlan p{};
  p.U = U;
  p.MT = (U >= 128 && g.B % 16 == 0) ? 128 : 64;
  const int NT = U / p.MT;
  int device = 0, smem_optin = 0;
  cudaError_t e = cudaGetDevice(&device);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, device);
  if (e != cudaSuccess) return e;
  const int mult = p.MT == 128 ? 16 : 8;
  auto two_stage_bytes = [&](int J_) {   // two stages of one item's operands, plus slack
    const int NR_ = (g.B * J_ + mult - 1) / mult * mult;
    const size_t item = (size_t)(split ? 2 : 1) * ((size_t)32 * U + (size_t)NR_ * (U + (J_ - 1) * p.MT) * 2);
    return 2 * (item + 127) / 128 * 128 + (size_t)NR_ * NR_ * 2 + 256 + 2048;
  };
  // tiles per group: enough that N = B*J reaches 16 columns, as long as two
  // stages of operands fit in shared memory
  int J = 1;
  while (J < NT && g.B * J < 16 && two_stage_bytes(2 * J) <= (size_t)smem_optin) J <<= 1;
  if (two_stage_bytes(J) > (size_t)smem_optin) return cudaErrorInvalidValue;
  p.J = J;
  p.NR = (g.B * J + mult - 1) / mult * mult;
  if (p.NR > 256) return cudaErrorInvalidValue;
  p.K = U + (J - 1) * p.MT;
  const int cols = (NT / J) * p.NR;
  if (cols > 512) return cudaErrorInvalidValue;
  p.split = split;
  // One item's operands (128-byte multiple); items per pass: enough that small
  // items share the smallest accumulator allocation (32 columns), within 64 KB.
  p.item_bytes = ((size_t)(split ? 2 : 1) * ((size_t)32 * U + (size_t)p.NR * p.K * 2) + 127) / 128 * 128;
  p.ipc = cols >= 32 ? 1 : 32 / cols;
  while (p.ipc > 1 && (size_t)p.ipc * p.item_bytes > 48 * 1024) p.ipc >>= 1;
  if (2 * p.ipc * cols > 512) return cudaErrorInvalidValue;
  // Two stages of operands, plus slack past the last one: a B-operand read
  // with its two strides exchanged would stay inside the allocation.
  p.smem = 2 * (size_t)p.ipc * p.item_bytes + (size_t)p.NR * p.NR * 2 + 256;
  const int cols_all = 2 * p.ipc * cols;        // two stages of accumulators
  p.tmem_cols = pow2_at_least(cols_all < 32 ? 32 : cols_all);
  int occ = 0;
  e = p.MT == 128 ? (split ? tc_occupancy<128, true>(p, device, &occ) : tc_occupancy<128, false>(p, device, &occ))
                  : (split ? tc_occupancy<64, true>(p, device, &occ) : tc_occupancy<64, false>(p, device, &occ));
  if (e != cudaSuccess) return e;
  // every resident CTA holds its accumulator columns for its whole life
  const int by_tmem = 512 / p.tmem_cols;
  const int per_sm = occ < by_tmem ? occ : by_tmem;
  if (per_sm < 1) return cudaErrorInvalidConfiguration;
  const long passes = ((long)g.M * g.D + p.ipc - 1) / p.ipc;
  long grid = (long)num_sms * per_sm;
  p.grid = (int)(grid > passes ? passes : grid);
  p.per_sm = per_sm;
  *out = p;
  return cudaSuccess;
}

cudaError_t launch_tile_tc(const Dims& g, float* state, const float* taps, const TcPlan& p, int i, int* err,
                           int wait_limit, cudaStream_t st) {
  if ((i & -i) != p.U || p.grid < 1) return cudaErrorInvalidValue;
  const int ow = is_pow2(i) ? 1 : 0;
  if (p.MT == 128) {
    if (p.split) k_tile_tc<128, true><<<p.grid, kTcThreads, p.smem, st>>>(g, state, taps, p, i, ow, err, wait_limit);
    else k_tile_tc<128, false><<<p.grid, kTcThreads, p.smem, st>>>(g, state, taps, p, i, ow, err, wait_limit);
  } else {
    if (p.split) k_tile_tc<64, true><<<p.grid, kTcThreads, p.smem, st>>>(g, state, taps, p, i, ow, err, wait_limit);
    else k_tile_tc<64, false><<<p.grid, kTcThreads, p.smem, st>>>(g, state, taps, p, i, ow, err, wait_limit);
  }
  return cudaGetLastError();
}

}  // namespace fi
