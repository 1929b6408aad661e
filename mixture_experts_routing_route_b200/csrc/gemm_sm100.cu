// Grouped expert GEMM on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// "MegaBlocks 01 - why MoE is hard", section 2 (the per-expert GEMMs are
// small, variable in M and skewed) and section 4.3 (bmm -> activation -> bmm
// over weights [E, hs, ffn]). Instead of padding every expert to a fixed
// capacity, the experts' rows are contiguous segments of one matrix and the
// kernel walks a device-side list of 128-row tiles, so M varies per expert
// with no host synchronisation and experts with no rows read no weights.
//
//   C[rows of e, n-tile] = epilogue( A[rows of e, :] . B[e][:, n-tile] )
//   A: [rows_max, K] bf16 row-major (K-major operand)
//   B: [E, K, N] bf16 row-major (MN-major operand; the pages' layout)
//   epilogue: SwiGLU (two B matrices, W_gate and W_up, side by side in one
//             N=256 MMA: silu(gate) * up), GELU (exact erf), or plain store;
//             fp32 in registers, rounded once to bf16.
//
// CTA = 6 warps, one CTA per SM, persistent over tiles:
//   warp 0   TMA producer: A tile 128x64 and B tile 64xN per stage, 128-byte
//            swizzle, into a 4-stage shared-memory ring (mbarrier full/empty)
//   warp 1   MMA issuer: one thread issues tcgen05.mma (M=128, N=256, K=16;
//            M=64 for a tile of at most 64 valid rows) into a double-buffered
//            fp32 accumulator in tensor memory and frees ring slots /
//            publishes accumulators with tcgen05.commit
//   warps 2-5 epilogue: tcgen05.ld of their 32-lane quarter of the
//            accumulator, activation, bf16 rows staged in shared memory and
//            stored as whole 128-byte segments, valid rows only
// Tiles are ordered expert-major, then N, with the M tile fastest, so CTAs
// that run at the same time share one weight column block through L2; a
// partial last wave is split into half-width tiles.
// Every wait is bounded; a time-out sets MOE_DEVERR_TIMEOUT and unwinds.
#include "common.cuh"
#include "ptx.cuh"
#include <cudaTypedefs.h>
#include <cmath>

namespace moe {

namespace {

constexpr int BM = 128;  // rows of A per CTA
constexpr int BK = 64;   // 64 bf16 = one 128-byte swizzle row
constexpr int kThreads = 192;
constexpr int kMaxE = 256;
constexpr int kBoxBytes = 64 * BK * 2;  // one 64-column B box: 8 KB

// EPI_COMBINE (down projection, k = 1): each row, rounded to bf16 as
// EPI_STORE would store it, is scaled by its slot's top-k weight in fp32
// (fmaf(w, y, 0), the combine's own arithmetic for one slot), rounded again
// and stored at its token's row of the layer output.
enum { EPI_SWIGLU = 0, EPI_GELU = 1, EPI_STORE = 2, EPI_COMBINE = 3 };

struct GemmArgs {
  const int32_t* seg;       // [E+1] row segment offsets
  __nv_bfloat16* out;       // [rows_max, N]
  const int32_t* row_slot;  // gathering A, or EPI_COMBINE: slot of each row (token = slot / k)
  const float* comb_w;      // EPI_COMBINE: top-k weight of each slot
  const int32_t* kept;      // [E] rows of each expert from seg[e] (binned layout), or null:
                            // seg[e + 1] - seg[e]
  int k;
  int E;
  int K;
  int N;  // output columns
  long long rows_max;
  long long slots;  // EPI_COMBINE: T * k (slot indices are checked against it)
  Control* ctl;
};

// silu(g) = g / (1 + e^-g) with the hardware exponential and reciprocal
// (CUDA's __expf and __fdividef intrinsics, a few ulp of fp32): the result is
// rounded to bf16 (2^-9 relative), so their error never shows, and the
// epilogue of the up projection runs in the tensor cores' shadow. For
// g < -88 the exponential overflows and __fdividef returns 0, the limit.
__device__ __forceinline__ float silu(float g) { return __fdividef(g, 1.0f + __expf(-g)); }
__device__ __forceinline__ float gelu_erf(float z) {
  return 0.5f * z * (1.0f + erff(z * 0.70710678118654752440f));
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// ------------------------------------------------------------------ schedule
// Warp 0: tile_start[e] = exclusive prefix of the per-expert unit counts
// ceil(m_e / TILE_M) * ntn (m_e = cnt[e] rows from seg[e]); tile_start[E] =
// total. Lane l owns experts [8l, 8l + 8). A segment whose rows are out of
// range is reported and gets zero tiles.
template <int TILE_M>
__device__ __forceinline__ void build_schedule(const GemmArgs& args, int ntn, const int* seg_s,
                                               const int* cnt_s, int* tile_start_s, int lane) {
  const int E = args.E;
  int loc[8];
  int sum = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane * 8 + i;
    int m = 0;
    if (e < E) {
      m = cnt_s[e];
      if (m < 0 || seg_s[e] < 0 || static_cast<long long>(seg_s[e]) + m > args.rows_max ||
          seg_s[e] + m > seg_s[e + 1]) {
        set_error(args.ctl, MOE_DEVERR_ROW_RANGE);
        m = 0;
      }
    }
    loc[i] = ((m + TILE_M - 1) / TILE_M) * ntn;
    sum += loc[i];
  }
  int incl = sum;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += n;
  }
  int run = incl - sum;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = lane * 8 + i;
    if (e < E) tile_start_s[e] = run;
    run += loc[i];
  }
  // The lanes cover experts 0..255 only; the total goes to entry E (which is
  // 256 when E = 256). Experts >= E contributed 0 tiles to the sum.
  if (lane == 31) tile_start_s[E] = incl;
}

// Tile -> (expert, first row, valid rows, first output column, half width).
struct Tile {
  int e, row0, rows, n0;
  bool half;
};

// Work units: tiles ordered expert-major, then N tile, M tile fastest, dealt
// round-robin to W persistent workers. When the last wave would leave workers
// idle (total % W = r tiles, 2r <= W), those r tiles become 2r half-width
// units (N/2 columns each), so the tail takes half a tile's time.
__device__ __forceinline__ bool split_tail(int total, int W) {
  const int r = total % W;
  return r != 0 && 2 * r <= W;
}

__device__ __forceinline__ int num_units(int total, int W) {
  return split_tail(total, W) ? total + total % W : total;
}

template <int TILE_M, int OUT_N>
__device__ __forceinline__ Tile decode_unit(int u, int total, int W, const int* tile_start,
                                            const int* seg, const int* cnt, int E) {
  int tau = u, half = -1;
  if (split_tail(total, W)) {
    const int r = total % W;
    if (u >= total - r) {
      const int h = u - (total - r);
      tau = total - r + (h >> 1);
      half = h & 1;
    }
  }
  int lo = 0, hi = E - 1;  // last e with tile_start[e] <= tau
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tile_start[mid] <= tau) lo = mid; else hi = mid - 1;
  }
  const int e = lo;
  const int m_e = cnt[e];
  const int mt_e = (m_e + TILE_M - 1) / TILE_M;
  const int local = tau - tile_start[e];
  const int nt = local / mt_e, mt = local - nt * mt_e;
  Tile t;
  t.e = e;
  t.row0 = seg[e] + mt * TILE_M;
  t.rows = min(TILE_M, m_e - mt * TILE_M);
  t.n0 = nt * OUT_N + (half > 0 ? OUT_N / 2 : 0);
  t.half = half >= 0;
  return t;
}

// ------------------------------------------------------------------ epilogue
// Epilogue of one warp through shared memory: for each 64-column group the
// warp writes its rows (thread = row, 2 x 64 bytes) into a padded staging
// buffer, then stores them back as whole 128-byte row segments, 8 lanes per
// row, 4 rows per store instruction. Only rows [0, nrows) of the warp are
// stored (rows past the expert's segment never are).
constexpr int kStageRow = 128 + 16;            // bytes per staged row (16 B pad: no bank conflicts)
constexpr int kStageWarpBytes = 32 * kStageRow;

template <int EPI, int OUTN>
__device__ __forceinline__ void epilogue_staged(uint32_t tbase, uint8_t* buf, const GemmArgs& args,
                                                long long row_base, int nrows, int N, int n0,
                                                int lane) {
  __nv_bfloat16* out = args.out;
  // EPI_COMBINE: this lane's row -> (token, weight); -1: nothing to store
  int tok = -1;
  float wgt = 0.f;
  if constexpr (EPI == EPI_COMBINE) {
    if (lane < nrows) {
      const int slot = __ldg(args.row_slot + row_base + lane);
      if (slot >= 0 && slot < args.slots) {
        tok = slot / args.k;
        wgt = __ldg(args.comb_w + slot);
      } else if (slot >= args.slots) {
        set_error(args.ctl, MOE_DEVERR_ROW_RANGE);
      }
    }
  }
#pragma unroll 1
  for (int g = 0; g < OUTN; g += 64) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int c = g + 32 * h;
      uint32_t v[32];
      uint32_t packed[16];
      if constexpr (EPI == EPI_SWIGLU) {
        uint32_t u[32];
        tmem_ld_32x32b_x32(tbase + c, v);
        tmem_ld_32x32b_x32(tbase + OUTN + c, u);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float h0 = silu(__uint_as_float(v[2 * i])) * __uint_as_float(u[2 * i]);
          const float h1 = silu(__uint_as_float(v[2 * i + 1])) * __uint_as_float(u[2 * i + 1]);
          packed[i] = pack_bf16(h0, h1);
        }
      } else {
        tmem_ld_32x32b_x32(tbase + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float a = __uint_as_float(v[2 * i]), b = __uint_as_float(v[2 * i + 1]);
          if (EPI == EPI_GELU) { a = gelu_erf(a); b = gelu_erf(b); }
          if (EPI == EPI_COMBINE) {
            a = fmaf(wgt, __bfloat162float(__float2bfloat16_rn(a)), 0.f);
            b = fmaf(wgt, __bfloat162float(__float2bfloat16_rn(b)), 0.f);
          }
          packed[i] = pack_bf16(a, b);
        }
      }
      uint4* sp = reinterpret_cast<uint4*>(buf + lane * kStageRow + 64 * h);
#pragma unroll
      for (int i = 0; i < 4; ++i)
        sp[i] = make_uint4(packed[4 * i], packed[4 * i + 1], packed[4 * i + 2], packed[4 * i + 3]);
    }
    __syncwarp();
    const int cq = lane & 7, rsub = lane >> 3;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int rr = it * 4 + rsub;
      long long dst = row_base + rr;
      if constexpr (EPI == EPI_COMBINE) dst = __shfl_sync(0xffffffffu, tok, rr);
      if (rr < nrows && dst >= 0) {
        const uint4 val = *reinterpret_cast<const uint4*>(buf + rr * kStageRow + cq * 16);
        *reinterpret_cast<uint4*>(out + static_cast<size_t>(dst) * N + n0 + g + cq * 8) = val;
      }
    }
    __syncwarp();
  }
}

// ==================================================================== kernel
// Tile 128 x NMMA per CTA, 4-stage ring of 48 KB (NMMA = 256). A tile with
// at most 64 valid rows (an expert's last) runs as an M = 64 MMA: half the
// tensor work, the same operand loads. In tensor memory an M = 64 result
// keeps rows 16 q .. 16 q + 15 in lanes 32 q .. 32 q + 15 (q = 0..3), so each
// epilogue warp still owns one lane quarter, with 16 rows in it.
constexpr int STAGES = 4;

template <int EPI, int NMMA>
struct Cfg {
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = BK * NMMA * 2;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int OUT_N = EPI == EPI_SWIGLU ? NMMA / 2 : NMMA;
  static constexpr int TMEM_COLS = 2 * NMMA;
  static constexpr size_t STAGING = 4 * kStageWarpBytes;  // epilogue staging, one per warp
  static constexpr size_t SMEM = static_cast<size_t>(STAGES) * STAGE_BYTES + STAGING + 1024;
};

// B boxes of one stage: SwiGLU puts NBOX/2 gate boxes then NBOX/2 up boxes
// over the same output columns.
template <int EPI, int NBOX>
__device__ __forceinline__ void load_b_boxes(uint8_t* sb, const CUtensorMap* b0,
                                             const CUtensorMap* b1, uint64_t* bar, int n0,
                                             int brow) {
#pragma unroll
  for (int j = 0; j < NBOX; ++j) {
    if constexpr (EPI == EPI_SWIGLU) {
      constexpr int H = NBOX / 2;
      tma_load_2d(sb + j * kBoxBytes, j < H ? b0 : b1, bar, n0 + (j % H) * 64, brow);
    } else {
      tma_load_2d(sb + j * kBoxBytes, b0, bar, n0 + j * 64, brow);
    }
  }
}

// GATHER: A is not a gathered copy but the token rows themselves: the
// producer warp loads each stage's 128 A rows with 32 tile::gather4 loads
// (lane l: rows 4l..4l+3, token row_slot[row] / k, one-row boxes), so the
// up projection reads x directly and x_perm is never written. Rows past the
// expert's segment load token 0 and are never stored.
template <int EPI, int NMMA, bool GATHER>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                const __grid_constant__ CUtensorMap tmB1, GemmArgs args) {
  pdl_begin();
  using C = Cfg<EPI, NMMA>;
  static_assert(!GATHER || (EPI != EPI_STORE && EPI != EPI_COMBINE), "only the up projection gathers");
  // A half-width unit still loads whole 64-column boxes: gate and up halves
  // need at least one box each under SwiGLU.
  static_assert(EPI == EPI_SWIGLU ? NMMA >= 256 : NMMA >= 128, "half units need whole boxes");
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES], empty_bar[STAGES];
  __shared__ __align__(8) uint64_t tfull_bar[2], tempty_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int seg_s[kMaxE + 1];
  __shared__ int cnt_s[kMaxE];
  __shared__ int tile_start_s[kMaxE + 1];
  __shared__ volatile int abort_s;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E;
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));

  for (int i = threadIdx.x; i <= E; i += kThreads) {
    seg_s[i] = __ldg(args.seg + i);
    if (i < E)
      cnt_s[i] = args.kept != nullptr ? __ldg(args.kept + i) : __ldg(args.seg + i + 1) - __ldg(args.seg + i);
  }
  if (threadIdx.x == 0) abort_s = 0;
  __syncthreads();
  if (warp == 0) build_schedule<BM>(args, args.N / C::OUT_N, seg_s, cnt_s, tile_start_s, lane);
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull_bar[b], 1); mbar_init(&tempty_bar[b], 4); }
    mbar_init(&drain_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(&tmem_base_s, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  const int total_tiles = tile_start_s[E];
  const int W = gridDim.x;
  const int total = num_units(total_tiles, W);
  const int nkb = args.K / BK;

  if (warp == 0 && !GATHER) {
    // One thread waits for each ring slot, arms it and issues its loads.
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB0);
      prefetch_tmap(&tmB1);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0;  // stages that ever received a load
      uint32_t last_parity = 0;  // parity of that stage's latest load
      for (int u = blockIdx.x; u < total && !abort_s; u += W) {
        const Tile t = decode_unit<BM, C::OUT_N>(u, total_tiles, W, tile_start_s, seg_s, cnt_s, E);
        const uint32_t tx = C::A_BYTES + (t.half ? C::B_BYTES / 2 : C::B_BYTES);
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u)) {
            set_error(args.ctl, MOE_DEVERR_TIMEOUT);
            abort_s = 1;
            break;
          }
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          mbar_arrive_expect_tx(&full_bar[stage], tx);
          tma_load_2d(sa, &tmA, &full_bar[stage], kb * BK, t.row0);
          const int brow = t.e * args.K + kb * BK;
          if (t.half)
            load_b_boxes<EPI, NMMA / 128>(sb, &tmB0, &tmB1, &full_bar[stage], t.n0, brow);
          else
            load_b_boxes<EPI, NMMA / 64>(sb, &tmB0, &tmB1, &full_bar[stage], t.n0, brow);
          issued_mask |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      // Every load issued must have landed before the CTA may exit.
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s)) if (!mbar_wait_bounded(&full_bar[s], (last_parity >> s) & 1u)) set_error(args.ctl, MOE_DEVERR_TIMEOUT);
    }
  } else if (warp == 0) {
    // GATHER: lane 0 waits for each ring slot and arms it, then the whole
    // warp issues its 32 gather4 loads (lane 0 also the B boxes).
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB0);
      prefetch_tmap(&tmB1);
    }
    int stage = 0;
    uint32_t phase = 0;
    uint32_t issued_mask = 0;
    uint32_t last_parity = 0;
    bool go = true;
    for (int u = blockIdx.x; u < total && go; u += W) {
      const Tile t = decode_unit<BM, C::OUT_N>(u, total_tiles, W, tile_start_s, seg_s, cnt_s, E);
      const uint32_t tx = C::A_BYTES + (t.half ? C::B_BYTES / 2 : C::B_BYTES);
      int tok[4] = {0, 0, 0, 0};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = lane * 4 + i;
        if (r < t.rows) tok[i] = __ldg(args.row_slot + t.row0 + r) / args.k;
      }
      for (int kb = 0; kb < nkb; ++kb) {
        int ok = 0;
        if (lane == 0) {
          ok = !abort_s && mbar_wait_bounded(&empty_bar[stage], phase ^ 1u);
          if (!ok && !abort_s) {
            set_error(args.ctl, MOE_DEVERR_TIMEOUT);
            abort_s = 1;
          }
          if (ok) mbar_arrive_expect_tx(&full_bar[stage], tx);
        }
        if (!__shfl_sync(0xffffffffu, ok, 0)) {
          go = false;
          break;
        }
        uint8_t* sa = smem + stage * C::STAGE_BYTES;
        uint8_t* sb = sa + C::A_BYTES;
        tma_gather4(sa + lane * 512, &tmA, &full_bar[stage], kb * BK, tok[0], tok[1], tok[2], tok[3]);
        if (lane == 0) {
          const int brow = t.e * args.K + kb * BK;
          if (t.half)
            load_b_boxes<EPI, NMMA / 128>(sb, &tmB0, &tmB1, &full_bar[stage], t.n0, brow);
          else
            load_b_boxes<EPI, NMMA / 64>(sb, &tmB0, &tmB1, &full_bar[stage], t.n0, brow);
        }
        issued_mask |= 1u << stage;
        last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
        if (++stage == STAGES) { stage = 0; phase ^= 1u; }
      }
    }
    if (lane == 0)
      for (int s = 0; s < STAGES; ++s)
        if (issued_mask & (1u << s)) if (!mbar_wait_bounded(&full_bar[s], (last_parity >> s) & 1u)) set_error(args.ctl, MOE_DEVERR_TIMEOUT);
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t kIdescFull = make_idesc_bf16(BM, NMMA);
      constexpr uint32_t kIdescHalf = make_idesc_bf16(BM, NMMA / 2);
      constexpr uint32_t kIdescFull64 = make_idesc_bf16(64, NMMA);
      constexpr uint32_t kIdescHalf64 = make_idesc_bf16(64, NMMA / 2);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued_any = false;
      for (int u = blockIdx.x; u < total && !abort_s; u += W) {
        const Tile t = decode_unit<BM, C::OUT_N>(u, total_tiles, W, tile_start_s, seg_s, cnt_s, E);
        const uint32_t idesc = t.rows <= 64 ? (t.half ? kIdescHalf64 : kIdescFull64)
                                            : (t.half ? kIdescHalf : kIdescFull);
        if (!mbar_wait_bounded(&tempty_bar[acc], acc_phase ^ 1u)) {
          set_error(args.ctl, MOE_DEVERR_TIMEOUT);
          abort_s = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * NMMA;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(&full_bar[stage], phase)) {
            set_error(args.ctl, MOE_DEVERR_TIMEOUT);
            abort_s = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t adesc = make_sw128_desc(a_addr + kk * 32, 16, 1024);
            const uint64_t bdesc = make_sw128_desc(b_addr + kk * 2048, kBoxBytes, 1024);
            umma_bf16(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          issued_any = true;
          umma_commit(&empty_bar[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull_bar[acc]);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (issued_any) {
        // Tensor memory is freed below: wait until every MMA issued is done.
        umma_commit(&drain_bar);
        (void)mbar_wait_bounded(&drain_bar, 0);
      }
    }
  } else {
    // epilogue warps 2..5: TMEM lane quarter = warp % 4
    const int q = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    for (int u = blockIdx.x; u < total; u += W) {
      // Lane 0 polls and decides for the whole warp, so the warp-wide
      // tcgen05.ld below always runs converged.
      int ok = 0;
      if (lane == 0) {
        ok = !abort_s && mbar_wait_bounded(&tfull_bar[acc], acc_phase);
        if (!ok && !abort_s) {
          set_error(args.ctl, MOE_DEVERR_TIMEOUT);
          abort_s = 1;
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      const Tile t = decode_unit<BM, C::OUT_N>(u, total_tiles, W, tile_start_s, seg_s, cnt_s, E);
      tc_fence_after();
      const bool m64 = t.rows <= 64;
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * NMMA;
      {
        uint8_t* buf = smem + STAGES * C::STAGE_BYTES + q * kStageWarpBytes;
        const int wrow = m64 ? q * 16 : q * 32;
        const int nrows = max(0, min(m64 ? 16 : 32, t.rows - wrow));
        if (t.half)
          epilogue_staged<EPI, C::OUT_N / 2>(tbase, buf, args, t.row0 + wrow, nrows, args.N, t.n0, lane);
        else
          epilogue_staged<EPI, C::OUT_N>(tbase, buf, args, t.row0 + wrow, nrows, args.N, t.n0, lane);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty_bar[acc]);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ============================================================ CTA-pair kernel
// The same grouped GEMM on tile pairs (cta_group::2): the two CTAs of a
// cluster compute one 256-row x NMMA tile together. CTA r loads A rows
// [row0 + 128 r, +128) and its half of the B columns (for SwiGLU: CTA 0 the
// W_gate box(es), CTA 1 the W_up box(es) of the same output columns) into a
// 6-stage ring of 32 KB; the even CTA issues M = 256 MMAs that read both CTAs'
// operands and write each CTA's 128 rows (all NMMA columns) into that CTA's
// tensor memory, so both epilogues see gate and up side by side as before.
// Per k-block an SM moves 32 KB into shared memory instead of 48 KB for the
// same tensor work: the fill bandwidth, not the tensor core, bounds the
// single-CTA kernel.
//
// Barriers: full[s] lives in the even CTA, armed there with both CTAs' bytes;
// both CTAs' TMA loads count their bytes on it (the cta_group::2 TMA form).
// empty[s] and tfull[acc] live in both CTAs; the MMA commits arrive on both
// (multicast). tempty[acc] lives in the even CTA and counts the 8 epilogue
// warps of the pair. Every wait is bounded; a time-out sets
// MOE_DEVERR_TIMEOUT and unwinds; the peer notices through its own bounded
// waits. Both CTAs meet at two cluster barriers only: after set-up and before
// tensor memory is freed, reached on every path.
//
// Work is handed out dynamically: the even CTA's producer takes the next unit
// from a counter in the control block (atomicAdd) when it is ready to load
// one and publishes it through a small ring in both CTAs' shared memory
// (unit_full in each CTA, unit_empty in the even CTA counting the ten readers:
// the peer's producer, the MMA thread and the pair's 8 epilogue warps); a
// value >= the unit count ends every role's loop. The units in flight thus
// stay a window of consecutive units, and the pairs sharing a weight block
// read it at nearly the same time (with a fixed round-robin deal the pairs
// drifted apart by up to a tile over a launch and re-read blocks from DRAM).
// The last pair to finish resets the counter for the next launch.
constexpr int kPairStages = 6;
constexpr int kPairRows = 256;
constexpr int kUnitSlots = 4;  // ring of work units published to the pair's roles
constexpr uint32_t kUnitReaders = 10;  // peer producer + MMA thread + 8 epilogue warps

template <int EPI>
struct PairCfg {
  static constexpr int NMMA = 256;
  static constexpr int A_BYTES = 128 * BK * 2;           // this CTA's 128 rows
  static constexpr int B_BYTES = BK * (NMMA / 2) * 2;     // this CTA's half of the columns
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;   // 32 KB
  static constexpr int OUT_N = EPI == EPI_SWIGLU ? NMMA / 2 : NMMA;
  static constexpr int TMEM_COLS = 2 * NMMA;
  static constexpr size_t STAGING = 4 * kStageWarpBytes;
  static constexpr size_t SMEM = static_cast<size_t>(kPairStages) * STAGE_BYTES + STAGING + 1024;
};

// This CTA's B boxes of one stage. Full unit: SwiGLU CTA 0 loads W_gate
// columns [n0, n0 + 128), CTA 1 the same W_up columns; otherwise CTA r loads
// columns [n0 + 128 r, +128). Half-width unit: one 64-column box each, W_gate
// / W_up at n0 (SwiGLU) or [n0 + 64 r, +64).
template <int EPI>
__device__ __forceinline__ void load_b_pair(uint8_t* sb, const CUtensorMap* b0, const CUtensorMap* b1,
                                            uint32_t bar, int n0, int brow, uint32_t rank, bool half) {
  if constexpr (EPI == EPI_SWIGLU) {
    const CUtensorMap* m = rank == 0 ? b0 : b1;
    tma_load_2d_pair(sb, m, bar, n0, brow);
    if (!half) tma_load_2d_pair(sb + kBoxBytes, m, bar, n0 + 64, brow);
  } else {
    if (half) {
      tma_load_2d_pair(sb, b0, bar, n0 + 64 * static_cast<int>(rank), brow);
    } else {
      const int c = n0 + 128 * static_cast<int>(rank);
      tma_load_2d_pair(sb, b0, bar, c, brow);
      tma_load_2d_pair(sb + kBoxBytes, b0, bar, c + 64, brow);
    }
  }
}

template <int EPI>
__global__ void __launch_bounds__(kThreads, 1)
grouped_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                  const __grid_constant__ CUtensorMap tmB1, GemmArgs args) {
  pdl_begin();
  using C = PairCfg<EPI>;
  constexpr int NMMA = C::NMMA;
  constexpr int STAGES_P = kPairStages;
  extern __shared__ uint8_t smem_raw[];
  __shared__ __align__(8) uint64_t full_bar[STAGES_P], empty_bar[STAGES_P];
  __shared__ __align__(8) uint64_t tfull_bar[2], tempty_bar[2], drain_bar;
  __shared__ uint32_t tmem_base_s;
  __shared__ int seg_s[kMaxE + 1];
  __shared__ int cnt_s[kMaxE];
  __shared__ int tile_start_s[kMaxE + 1];
  __shared__ volatile int abort_s;
  __shared__ __align__(8) uint64_t unit_full[kUnitSlots], unit_empty[kUnitSlots];
  __shared__ volatile int unit_ring[kUnitSlots];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int E = args.E;
  const uint32_t rank = cluster_ctarank();  // 0: the CTA that issues the MMAs
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));

  for (int i = threadIdx.x; i <= E; i += kThreads) {
    seg_s[i] = __ldg(args.seg + i);
    if (i < E)
      cnt_s[i] = args.kept != nullptr ? __ldg(args.kept + i) : __ldg(args.seg + i + 1) - __ldg(args.seg + i);
  }
  if (threadIdx.x == 0) abort_s = 0;
  __syncthreads();
  if (warp == 0) build_schedule<kPairRows>(args, args.N / C::OUT_N, seg_s, cnt_s, tile_start_s, lane);
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES_P; ++s) { mbar_init(&full_bar[s], 1); mbar_init(&empty_bar[s], 1); }
    for (int b = 0; b < 2; ++b) { mbar_init(&tfull_bar[b], 1); mbar_init(&tempty_bar[b], 8); }
    for (int i = 0; i < kUnitSlots; ++i) {
      mbar_init(&unit_full[i], 1);
      mbar_init(&unit_empty[i], kUnitReaders);
    }
    mbar_init(&drain_bar, 1);
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc_pair(&tmem_base_s, C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers initialised and tensor memory allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = tmem_base_s;
  const int total_tiles = tile_start_s[E];
  const int W = gridDim.x >> 1;  // pairs
  const int total = num_units(total_tiles, W);
  const int nkb = args.K / BK;
  // the even CTA's full, tempty and unit_empty barriers, as shared::cluster addresses
  const uint32_t full0 = mapa_shared(smem_u32(&full_bar[0]), 0);
  const uint32_t tempty0 = mapa_shared(smem_u32(&tempty_bar[0]), 0);
  const uint32_t uempty0 = mapa_shared(smem_u32(&unit_empty[0]), 0);

  // A reader's next unit: wait for its slot, read it, free the slot for the
  // producer (every reader frees every slot it reads, the end marker too).
  // Returns total (the end) on a time-out.
  auto next_unit = [&](int& uslot, uint32_t& uphase) -> int {
    int u = total;
    if (mbar_wait_cluster_bounded(&unit_full[uslot], uphase)) {
      u = unit_ring[uslot];
      mbar_arrive_cluster(uempty0 + uslot * 8u);
    } else {
      set_error(args.ctl, MOE_DEVERR_TIMEOUT);
      abort_s = 1;
    }
    if (++uslot == kUnitSlots) { uslot = 0; uphase ^= 1u; }
    return u < total ? u : total;
  };

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB0);
      prefetch_tmap(&tmB1);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued_mask = 0;  // stages that ever received a load
      uint32_t last_parity = 0;  // parity of that stage's latest load
      int uslot = 0;
      uint32_t uphase = 0;
      const uint32_t ring_peer = mapa_shared(smem_u32(const_cast<int*>(&unit_ring[0])), 1);
      const uint32_t ufull_peer = mapa_shared(smem_u32(&unit_full[0]), 1);
      // The even CTA takes units one ahead: the counter's round trip overlaps
      // the current unit's loads.
      auto take = [&]() -> int {
        return abort_s ? total
                       : static_cast<int>(min(atomicAdd(&args.ctl->gemm_next, 1u),
                                              static_cast<unsigned>(total)));
      };
      int u_next = rank == 0 ? take() : total;
      for (;;) {
        int u = total;
        if (rank == 0) {
          // publish the unit taken to both CTAs' readers
          if (!mbar_wait_cluster_bounded(&unit_empty[uslot], uphase ^ 1u)) {
            set_error(args.ctl, MOE_DEVERR_TIMEOUT);
            abort_s = 1;
            break;
          }
          u = abort_s ? total : u_next;
          if (u < total) u_next = take();
          unit_ring[uslot] = u;
          st_shared_cluster_u32(ring_peer + uslot * 4u, static_cast<uint32_t>(u));
          mbar_arrive(&unit_full[uslot]);
          mbar_arrive_cluster(ufull_peer + uslot * 8u);
          if (++uslot == kUnitSlots) { uslot = 0; uphase ^= 1u; }
        } else {
          u = next_unit(uslot, uphase);
        }
        if (u >= total || abort_s) break;
        const Tile t = decode_unit<kPairRows, C::OUT_N>(u, total_tiles, W, tile_start_s, seg_s, cnt_s, E);
        const uint32_t tx = 2u * (C::A_BYTES + (t.half ? C::B_BYTES / 2 : C::B_BYTES));
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_bounded(&empty_bar[stage], phase ^ 1u)) {
            set_error(args.ctl, MOE_DEVERR_TIMEOUT);
            abort_s = 1;
            break;
          }
          uint8_t* sa = smem + stage * C::STAGE_BYTES;
          uint8_t* sb = sa + C::A_BYTES;
          if (rank == 0) mbar_arrive_expect_tx(&full_bar[stage], tx);
          const uint32_t fb = full0 + stage * 8u;
          tma_load_2d_pair(sa, &tmA, fb, kb * BK, t.row0 + 128 * static_cast<int>(rank));
          load_b_pair<EPI>(sb, &tmB0, &tmB1, fb, t.n0, t.e * args.K + kb * BK, rank, t.half);
          issued_mask |= 1u << stage;
          last_parity = (last_parity & ~(1u << stage)) | (phase << stage);
          if (++stage == STAGES_P) { stage = 0; phase ^= 1u; }
        }
      }
      // Every load issued must have been consumed by the MMAs (so it landed)
      // before this CTA may leave: the MMA commit of each stage's last load
      // arrives on empty[s] in both CTAs.
      for (int s = 0; s < STAGES_P; ++s)
        if (issued_mask & (1u << s)) if (!mbar_wait_bounded(&empty_bar[s], (last_parity >> s) & 1u)) set_error(args.ctl, MOE_DEVERR_TIMEOUT);
      // The last pair to finish resets the unit counter for the next launch
      // (every pair's last take precedes its increment here).
      if (rank == 0 && atomicAdd(&args.ctl->gemm_done, 1u) == static_cast<unsigned>(W) - 1u) {
        atomicExch(&args.ctl->gemm_next, 0u);
        atomicExch(&args.ctl->gemm_done, 0u);
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      constexpr uint32_t kIdescFull = make_idesc_bf16(kPairRows, NMMA);
      constexpr uint32_t kIdescHalf = make_idesc_bf16(kPairRows, NMMA / 2);
      int stage = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool issued_any = false;
      int uslot = 0;
      uint32_t uphase = 0;
      for (;;) {
        const int u = next_unit(uslot, uphase);
        if (u >= total || abort_s) break;
        const Tile t = decode_unit<kPairRows, C::OUT_N>(u, total_tiles, W, tile_start_s, seg_s, cnt_s, E);
        const uint32_t idesc = t.half ? kIdescHalf : kIdescFull;
        if (!mbar_wait_cluster_bounded(&tempty_bar[acc], acc_phase ^ 1u)) {
          set_error(args.ctl, MOE_DEVERR_TIMEOUT);
          abort_s = 1;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * NMMA;
        bool ok = true;
        for (int kb = 0; kb < nkb; ++kb) {
          if (!mbar_wait_cluster_bounded(&full_bar[stage], phase)) {
            set_error(args.ctl, MOE_DEVERR_TIMEOUT);
            abort_s = 1;
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + stage * C::STAGE_BYTES);
          const uint32_t b_addr = a_addr + C::A_BYTES;
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t adesc = make_sw128_desc(a_addr + kk * 32, 16, 1024);
            const uint64_t bdesc = make_sw128_desc(b_addr + kk * 2048, kBoxBytes, 1024);
            umma_bf16_pair(d_tmem, adesc, bdesc, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          issued_any = true;
          umma_commit_pair_mc(&empty_bar[stage], 0x3);
          if (++stage == STAGES_P) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair_mc(&tfull_bar[acc], 0x3);
        if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
      }
      if (issued_any) {
        // Tensor memory is freed below: wait until every MMA issued is done.
        umma_commit_pair_mc(&drain_bar, 0x1);
        (void)mbar_wait_bounded(&drain_bar, 0);
      }
    }
  } else {
    // epilogue warps 2..5: TMEM lane quarter = warp % 4 of this CTA's 128 rows
    const int q = warp & 3;
    int acc = 0;
    uint32_t acc_phase = 0;
    int uslot = 0;
    uint32_t uphase = 0;
    for (;;) {
      int ok = 0, u = total;
      if (lane == 0) {
        u = next_unit(uslot, uphase);
        ok = u < total && !abort_s && mbar_wait_cluster_bounded(&tfull_bar[acc], acc_phase);
        if (!ok && u < total && !abort_s) {
          set_error(args.ctl, MOE_DEVERR_TIMEOUT);
          abort_s = 1;
        }
      }
      if (!__shfl_sync(0xffffffffu, ok, 0)) break;
      u = __shfl_sync(0xffffffffu, u, 0);
      const Tile t = decode_unit<kPairRows, C::OUT_N>(u, total_tiles, W, tile_start_s, seg_s, cnt_s, E);
      tc_fence_after();
      const uint32_t tbase = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * NMMA;
      {
        uint8_t* buf = smem + STAGES_P * C::STAGE_BYTES + q * kStageWarpBytes;
        const int crow = 128 * static_cast<int>(rank) + q * 32;  // first row of this warp in the tile
        const int nrows = max(0, min(32, t.rows - crow));
        if (t.half)
          epilogue_staged<EPI, C::OUT_N / 2>(tbase, buf, args, t.row0 + crow, nrows, args.N, t.n0, lane);
        else
          epilogue_staged<EPI, C::OUT_N>(tbase, buf, args, t.row0 + crow, nrows, args.N, t.n0, lane);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0 + acc * 8u);
      if (++acc == 2) { acc = 0; acc_phase ^= 1u; }
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no peer still reads or signals this CTA; every MMA is done
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

// ----------------------------------------------------------------- host side
}  // namespace

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    cudaDriverEntryPointQueryResult q;
    void* p = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2-D bf16 map over [rows, cols] with a row stride of ld elements, box
// [box_rows, 64 cols], 128-B swizzle.
bool make_tma_2d_bf16_ld(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols, uint64_t ld,
                         uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D bf16 map over [rows, cols] row-major (cols * 2 a multiple of 16), box
// [box_rows, box_cols], no swizzle: a box lands as box_rows rows of
// box_cols * 2 bytes, back to back.
bool make_tma_2d_bf16_plain(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                            uint32_t box_cols, uint32_t box_rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                        box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// 2-D bf16 map over [rows, cols] row-major, box [box_rows, 64 cols], 128-B swizzle.
bool make_tma_2d_bf16(CUtensorMap* m, const void* base, uint64_t rows, uint64_t cols,
                      uint32_t box_rows) {
  return make_tma_2d_bf16_ld(m, base, rows, cols, cols, box_rows);
}

namespace {

// A: [a_rows, K] row-major; a_rows = rows_max, or T when gathering (then
// row_slot / k pick each row's token).
template <int EPI, int NMMA, bool GATHER>
cudaError_t run_gemm(const void* A, int64_t a_rows, const int32_t* row_slot, int k, const void* B0,
                     const void* B1, int64_t rows_max, int K, int N, int E, const int32_t* seg,
                     const int32_t* kept, void* out, Control* ctl, cudaStream_t s,
                     const float* comb_w = nullptr, long long slots = 0) {
  using C = Cfg<EPI, NMMA>;
  CUtensorMap ta, tb0, tb1;
  if (!make_tma_2d_bf16(&ta, A, static_cast<uint64_t>(a_rows), K, GATHER ? 1 : BM))
    return cudaErrorInvalidValue;
  if (!make_tma_2d_bf16(&tb0, B0, static_cast<uint64_t>(E) * K, N, BK)) return cudaErrorInvalidValue;
  if (!make_tma_2d_bf16(&tb1, B1 ? B1 : B0, static_cast<uint64_t>(E) * K, N, BK)) return cudaErrorInvalidValue;
  GemmArgs a;
  a.seg = seg;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.row_slot = row_slot;
  a.kept = kept;
  a.k = k;
  a.E = E;
  a.K = K;
  a.N = N;
  a.rows_max = rows_max;
  a.comb_w = comb_w;
  a.slots = slots;
  a.ctl = ctl;
  auto kern = grouped_gemm_tc<EPI, NMMA, GATHER>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::SMEM));
  return launch_pdl(kern, dim3(num_sms()), dim3(kThreads), C::SMEM, s, false, ta, tb0, tb1, a);
}

// The CTA-pair kernel, for NMMA = 256. Each CTA's A box is 128 rows.
template <int EPI>
cudaError_t run_gemm_pair(const void* A, int64_t a_rows, const int32_t* row_slot, int k,
                          const void* B0, const void* B1, int64_t rows_max, int K, int N, int E,
                          const int32_t* seg, const int32_t* kept, void* out, Control* ctl,
                          cudaStream_t s, const float* comb_w = nullptr, long long slots = 0) {
  using C = PairCfg<EPI>;
  CUtensorMap ta, tb0, tb1;
  if (!make_tma_2d_bf16(&ta, A, static_cast<uint64_t>(a_rows), K, 128)) return cudaErrorInvalidValue;
  if (!make_tma_2d_bf16(&tb0, B0, static_cast<uint64_t>(E) * K, N, BK)) return cudaErrorInvalidValue;
  if (!make_tma_2d_bf16(&tb1, B1 ? B1 : B0, static_cast<uint64_t>(E) * K, N, BK)) return cudaErrorInvalidValue;
  GemmArgs a;
  a.seg = seg;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.row_slot = row_slot;
  a.kept = kept;
  a.k = k;
  a.E = E;
  a.K = K;
  a.N = N;
  a.rows_max = rows_max;
  a.comb_w = comb_w;
  a.slots = slots;
  a.ctl = ctl;
  auto kern = grouped_gemm_pair<EPI>;
  cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(C::SMEM));
  const int pairs = num_sms() / 2;
  return launch_pdl_cluster(kern, dim3(2 * pairs), dim3(kThreads), C::SMEM, s, 2, ta, tb0, tb1, a);
}

// Experts averaging at least this many rows run on CTA pairs (256-row tiles):
// below it the 256-row tile's padding costs more than the pair saves. The
// average is taken over the slots the permute distributes (T * k for a layer
// forward, whatever the row layout), so the dense and the binned layouts pick
// the same kernel. Measured on B200 (event medians, L2 evicted): at 1024 rows
// per expert the pair takes the down projection from 884 to 783 us and the up
// projection from 1528 to 1505 us; on a Zipf-skewed layer with 512 slots per
// expert and capacity 512 it is slower (up 90 vs 70 us, down 57 vs 45 us).
constexpr int64_t kPairMinRowsPerExpert = 768;

bool use_pair(int64_t slots, int E, int out_cols) {
  return out_cols % 256 == 0 && slots >= kPairMinRowsPerExpert * E;
}

template <bool GATHER>
cudaError_t run_up(const void* a, int64_t a_rows, const int32_t* row_slot, int k, const void* w1,
                   const void* w3, moe_act_t act, int64_t rows_max, int d, int F, int E,
                   const int32_t* seg, const int32_t* kept, void* h, Control* ctl,
                   cudaStream_t s, int64_t slots) {
  if (!GATHER && use_pair(slots, E, F)) {
    if (act == MOE_ACT_SWIGLU)
      return run_gemm_pair<EPI_SWIGLU>(a, a_rows, nullptr, k, w1, w3, rows_max, d, F, E, seg, kept, h,
                                       ctl, s);
    return run_gemm_pair<EPI_GELU>(a, a_rows, nullptr, k, w1, nullptr, rows_max, d, F, E, seg, kept, h,
                                   ctl, s);
  }
  if (act == MOE_ACT_SWIGLU)
    return run_gemm<EPI_SWIGLU, 256, GATHER>(a, a_rows, row_slot, k, w1, w3, rows_max, d, F, E, seg,
                                             kept, h, ctl, s);
  if (F % 256 == 0)
    return run_gemm<EPI_GELU, 256, GATHER>(a, a_rows, row_slot, k, w1, nullptr, rows_max, d, F, E,
                                           seg, kept, h, ctl, s);
  return run_gemm<EPI_GELU, 128, GATHER>(a, a_rows, row_slot, k, w1, nullptr, rows_max, d, F, E, seg,
                                         kept, h, ctl, s);
}

}  // namespace

cudaError_t launch_ffn_bf16(const void* a, int64_t a_rows, const int32_t* row_slot, int k,
                            const void* w1, const void* w3, const void* w2, moe_act_t act,
                            int64_t rows_max, int d, int F, int E, const int32_t* seg,
                            const int32_t* kept, void* h, void* y, Control* ctl, cudaStream_t s,
                            cudaEvent_t after_up, const CombineOut* comb, int64_t slots) {
  if (slots < 0) slots = rows_max;
  if (rows_max <= 0) {
    if (after_up) cudaEventRecord(after_up, s);
    return cudaSuccess;
  }
  cudaError_t err =
      row_slot != nullptr
          ? run_up<true>(a, a_rows, row_slot, k, w1, w3, act, rows_max, d, F, E, seg, kept, h, ctl, s,
                         slots)
          : run_up<false>(a, rows_max, nullptr, 1, w1, w3, act, rows_max, d, F, E, seg, kept, h, ctl,
                          s, slots);
  if (err != cudaSuccess) return err;
  if (after_up) cudaEventRecord(after_up, s);
  if (comb != nullptr) {  // k = 1: the combine in the down projection's epilogue
    const long long comb_slots = static_cast<long long>(comb->T) * k;
    if (use_pair(slots, E, d))
      return run_gemm_pair<EPI_COMBINE>(h, rows_max, comb->row_slot, k, w2, nullptr, rows_max, F, d, E,
                                        seg, kept, comb->out, ctl, s, comb->w, comb_slots);
    if (d % 256 == 0)
      return run_gemm<EPI_COMBINE, 256, false>(h, rows_max, comb->row_slot, k, w2, nullptr, rows_max, F,
                                               d, E, seg, kept, comb->out, ctl, s, comb->w, comb_slots);
    return run_gemm<EPI_COMBINE, 128, false>(h, rows_max, comb->row_slot, k, w2, nullptr, rows_max, F,
                                             d, E, seg, kept, comb->out, ctl, s, comb->w, comb_slots);
  }
  if (use_pair(slots, E, d))
    err = run_gemm_pair<EPI_STORE>(h, rows_max, nullptr, 1, w2, nullptr, rows_max, F, d, E, seg, kept,
                                   y, ctl, s);
  else if (d % 256 == 0)
    err = run_gemm<EPI_STORE, 256, false>(h, rows_max, nullptr, 1, w2, nullptr, rows_max, F, d, E,
                                          seg, kept, y, ctl, s);
  else
    err = run_gemm<EPI_STORE, 128, false>(h, rows_max, nullptr, 1, w2, nullptr, rows_max, F, d, E,
                                          seg, kept, y, ctl, s);
  return err;
}

}  // namespace moe
