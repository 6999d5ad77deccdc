// Persistent, warp-specialized tcgen05 GEMM for sm_100a.
//
//   warp 0      : TMA producer (one elected lane) filling a STAGES-deep ring of
//                 128B-swizzled A/B tiles in shared memory
//   warp 1      : TMEM allocator + MMA issuer (one lane issues tcgen05.mma,
//                 128 x BN x 16 per instruction, fp32 accumulator in TMEM)
//   warps 2..   : epilogue, 8 warps for bf16 outputs (4 for fp32); warp w
//                 reads TMEM lanes 32*(w%4)..+31 (its rows) -- two warps share
//                 a lane quarter and take alternate 32-column chunks -- applies
//                 the fused epilogue, writes the 32x32 chunk into swizzled
//                 shared memory and hands it to a TMA bulk tensor store (or
//                 fp32 reduce-add), double-buffered
//
// Two accumulator buffers in TMEM (2*BN columns) let the epilogue of tile i
// overlap the main loop of tile i+1.  Tiles are 128 x BN x 64; split-K (for
// the long-K weight-gradient GEMMs) adds fp32 partial sums with TMA reduce-add.
#include <algorithm>
#include <atomic>
#include <mutex>

#include "gemm_sm100.cuh"
#include "sm100_ptx.cuh"


namespace qat {

namespace {

constexpr int BM = 128;
constexpr int BK = 64;

// PAIR: the CTA pair of a 2-CTA cluster computes a 256 x BN tile with
// tcgen05 cta_group::2; each CTA stages 128 rows of A and BN/2 rows of B.
// Epilogues that read a bf16 tensor of the output's shape (residual or saved
// pre-activation) bring it in by TMA ahead of use (R).  bf16-output epilogues
// run 8 warps (their HBM traffic per FLOP is high: a lone warp per lane
// quarter left the tensor pipe idle), the fp32 split-K ones 4.
// FB (fused quantizing B producer): B is not loaded by TMA.  Each CTA keeps
// the B_ROWS x K slice of the current N block resident in shared memory as a
// panel of KBP k-blocks, written by the epilogue warps straight from the fp32
// weight (row amax, scale, codes, dequantized value, bf16) whenever the CTA's
// run of tiles enters a new N block; only A streams through the ring.
template <int BN, bool PAIR, int EPI, bool FB = false>
struct Cfg {
  static constexpr bool F32 = (EPI == EPI_F32 || EPI == EPI_F32_ATOMIC);
  static constexpr bool HAS_R = epi_reads_r(EPI);
  static constexpr bool ACT = epi_act_fwd(EPI);
  static constexpr int EW = F32 ? 4 : (FB && (ACT || HAS_R)) ? 4 : 8;  // epilogue warps
  static constexpr int THREADS = 64 + 32 * EW;
  static constexpr int B_ROWS = PAIR ? BN / 2 : BN;  // B rows staged by one CTA
  static constexpr int TILE_M = PAIR ? 2 * BM : BM;
  static constexpr int A_BYTES = BM * BK * 2;
  static constexpr int B_BYTES = FB ? 0 : B_ROWS * BK * 2;  // B bytes per ring stage
  // FB panel: KBP k-blocks of B_ROWS rows x 128 bytes (K <= 64 * KBP)
  static constexpr int KBP = !FB ? 0 : B_ROWS >= 128 ? 8 : B_ROWS >= 80 ? 10 : 16;
  static constexpr int KB_BYTES = B_ROWS * 128;
  static constexpr int PANEL_BYTES = KBP * KB_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int TMEM_COLS = (2 * BN <= 256) ? 256 : 512;  // a power of two >= 2*BN
  // per epilogue warp: two buffers of one or two 32x32 output chunks
  static constexpr int WBUF = (F32 || ACT) ? 8192 : 4096;
  static constexpr int STAGING_BYTES = EW * WBUF;
  static constexpr int R_BUFS = (EW == 8 || FB) ? 2 : 4;  // R chunks in flight per epilogue warp
  static constexpr int R_BYTES = HAS_R ? EW * R_BUFS * 2048 : 0;
  static constexpr int BAR_BYTES = 512;
  static constexpr int FIXED = PANEL_BYTES + STAGING_BYTES + R_BYTES + BAR_BYTES + 1024;
  static constexpr int STAGES_FIT = (232448 - FIXED) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 6 ? 6 : STAGES_FIT;
  static constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + FIXED;
  static_assert(STAGES >= 3, "pipeline too shallow");
  static_assert(KB_BYTES % 1024 == 0, "panel k-blocks must keep the 1024-byte swizzle atoms aligned");
  // barriers (full/empty per stage, tfull/tempty x2, mma_done, panel_full, R
  // ring per epilogue warp) followed by tmem_slot, abort flag and two ring positions
  static_assert((2 * STAGES + 6 + EW * R_BUFS) * 8 + 16 <= BAR_BYTES, "barrier block overflow");
  // FB conversion: rows per pass (float4 loads in flight per lane: RP * KBP / 2)
  static constexpr int RP = KBP > 10 ? 2 : 4;
  static_assert(RP >= 1, "conversion rows per pass");
};

struct KArgs {
  int M, N;
  int num_m_blk, num_n_blk, splits, kblk_total, kblk_per_split, num_tiles;
  void* D;
  int64_t ldd;
  void* D2;
  int64_t ldd2;
  const __nv_bfloat16* R;
  int64_t ldr;
  int accumulate;
  int* err;
  const float* W;  // FB: fp32 weight [N, K] row-major, quantized in the producer
  int K;           // FB: reduction length
  int bits;        // FB: grid (5, 6 or 8)
};

__device__ __forceinline__ float bf2f(__nv_bfloat16 x) { return __bfloat162float(x); }

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);  // .x = a (low half), .y = b
  return *reinterpret_cast<uint32_t*>(&v);
}

// Epilogue of one 32-column chunk of one row (this lane's), staged into the
// warp's shared-memory chunk buffers:
//   bf16 outputs: 32 rows x 64 B, 16-byte groups swizzled as TMA's 64-byte
//                 swizzle expects (group j of row r at j ^ ((r >> 1) & 3));
//   fp32 outputs: 32 rows x 128 B, 128-byte swizzle (group j at j ^ (r & 7)).
// Both patterns make each quarter-warp's 16-byte stores hit distinct banks.
template <int EPI>
__device__ __forceinline__ void stage_chunk(const KArgs& p, const uint32_t (&acc)[32],
                                            const uint4 (&rin)[4], uint32_t buf0, uint32_t buf1,
                                            int lane) {
  const float* v = reinterpret_cast<const float*>(acc);
  if constexpr (EPI == EPI_F32 || EPI == EPI_F32_ATOMIC) {
    const uint32_t row = buf0 + static_cast<uint32_t>(lane) * 128u;
#pragma unroll
    for (int j = 0; j < 8; ++j)
      st_shared_v4(row + ((static_cast<uint32_t>(j ^ (lane & 7))) << 4), acc[4 * j],
                   acc[4 * j + 1], acc[4 * j + 2], acc[4 * j + 3]);
  } else {
    const uint32_t off = static_cast<uint32_t>(lane) * 64u;
    const int sw = (lane >> 1) & 3;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float o[8];
      const __nv_bfloat16* r = reinterpret_cast<const __nv_bfloat16*>(&rin[j]);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float a = v[8 * j + i];
        if constexpr (EPI == EPI_BF16) {
          o[i] = a;
        } else if constexpr (EPI == EPI_BF16_RESID) {
          o[i] = __fadd_rn(a, bf2f(r[i]));
        } else if constexpr (EPI == EPI_DRELU2) {
          o[i] = __fmul_rn(__fmul_rn(a, fmaxf(bf2f(r[i]), 0.0f)), 2.0f);
        } else if constexpr (EPI == EPI_DLRELU2) {
          // d/dx leaky(x, 0.5)^2 = 2x (x > 0), x/2 (x <= 0): the scalings are exact
          const float pre = bf2f(r[i]);
          o[i] = __fmul_rn(a, pre > 0.0f ? __fmul_rn(pre, 2.0f) : __fmul_rn(pre, 0.5f));
        } else if constexpr (EPI == EPI_LRELU2) {  // buf1 <- leaky_relu(acc, 0.5)^2
          const float t = a > 0.0f ? a : __fmul_rn(a, 0.5f);
          o[i] = __fmul_rn(t, t);
        } else {  // EPI_RELU2: buf0 <- pre (when kept), buf1 <- relu(acc)^2
          const float t = fmaxf(a, 0.0f);
          o[i] = __fmul_rn(t, t);
        }
      }
      const uint32_t at = off + (static_cast<uint32_t>(j ^ sw) << 4);
      if constexpr (epi_act_fwd(EPI)) {
        st_shared_v4(buf0 + at, pack_bf16(v[8 * j], v[8 * j + 1]), pack_bf16(v[8 * j + 2], v[8 * j + 3]),
                     pack_bf16(v[8 * j + 4], v[8 * j + 5]), pack_bf16(v[8 * j + 6], v[8 * j + 7]));
        st_shared_v4(buf1 + at, pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]),
                     pack_bf16(o[6], o[7]));
      } else {
        st_shared_v4(buf0 + at, pack_bf16(o[0], o[1]), pack_bf16(o[2], o[3]), pack_bf16(o[4], o[5]),
                     pack_bf16(o[6], o[7]));
      }
    }
  }
}

__device__ __forceinline__ float absmax4(float4 v) {
  return fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w)));
}

// FB producer: fill this CTA's panel with the STE operand of weight rows
// n_base .. n_base + B_ROWS - 1, the training quantizer's arithmetic exactly:
//   amax = max(max_j |W_nj|, 1e-12), s = fl32(amax / L) (L = 127, or 15 for
//   int5), c = the grid's code of fl32(w / s), operand = bf16_rne(fl32(c * s)).
// Row r of k-block kb lands at kb * KB_BYTES + r * 128, its 16-byte group g
// (8 consecutive k) at g ^ (r & 7): the 128-byte-swizzled K-major layout a TMA
// load of the same tile would write.  Rows >= N and columns >= K are zero.
// Warp ew takes rows ew, ew + EW, ...; RP rows per pass keep RP * KBP / 2
// 16-byte loads in flight per lane.
template <class C, int BITS>
__device__ __forceinline__ void convert_panel(const KArgs& p, uint8_t* panel, int n_base, int ew,
                                              int lane) {
  constexpr int V = C::KBP / 2;  // float4 per lane per row (32 lanes x 4 floats per 128 columns)
  const int K4 = p.K >> 2;
  const int slots = p.kblk_total * 16;  // float4 slots of a panel row
  const float levels = grid_levels(BITS);
  const uint32_t pbase = smem_u32(panel);
#pragma unroll 1
  for (int r0 = ew; r0 < C::B_ROWS; r0 += C::RP * C::EW) {
    float4 v[C::RP][V];
    float amax[C::RP];
#pragma unroll
    for (int h = 0; h < C::RP; ++h) {
      const int r = r0 + h * C::EW;
      const int n = n_base + r;
      const bool valid = r < C::B_ROWS && n < p.N;
      const float4* row = reinterpret_cast<const float4*>(p.W + static_cast<int64_t>(valid ? n : 0) * p.K);
      amax[h] = 0.0f;
#pragma unroll
      for (int i = 0; i < V; ++i) {
        const int j = lane + 32 * i;
        v[h][i] = make_float4(0.f, 0.f, 0.f, 0.f);
        if (valid && j < K4) {
          v[h][i] = __ldg(row + j);
          amax[h] = fmaxf(amax[h], absmax4(v[h][i]));
        }
      }
    }
#pragma unroll
    for (int h = 0; h < C::RP; ++h) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1)
        amax[h] = fmaxf(amax[h], __shfl_xor_sync(0xffffffffu, amax[h], o));
    }
#pragma unroll
    for (int h = 0; h < C::RP; ++h) {
      const int r = r0 + h * C::EW;
      if (r >= C::B_ROWS) break;  // warp-uniform
      const float sc = div_rn(fmaxf(amax[h], 1e-12f), levels);
      const float rs = __frcp_rn(sc);
      const uint32_t rbase = pbase + static_cast<uint32_t>(r) * 128u;
      const uint32_t sw = static_cast<uint32_t>(r & 7);
#pragma unroll
      for (int i = 0; i < V; ++i) {
        const int j = lane + 32 * i;
        if (j < slots) {
          const float4 w = v[h][i];
          // the training quantizer's codes (exact float values) and fl32(c * s)
          const float2 s2 = make_float2(sc, sc);
          const float2 w01 = mul2(grid_code_values2<BITS>(w.x, w.y, sc, rs), s2);
          const float2 w23 = mul2(grid_code_values2<BITS>(w.z, w.w, sc, rs), s2);
          const uint32_t lo = pack_bf16(w01.x, w01.y);
          const uint32_t hi = pack_bf16(w23.x, w23.y);
          const uint32_t kb = static_cast<uint32_t>(j >> 4), g = static_cast<uint32_t>((j & 15) >> 1);
          st_shared_v2(rbase + kb * C::KB_BYTES + ((g ^ sw) << 4) + static_cast<uint32_t>(j & 1) * 8u,
                       lo, hi);
        }
      }
    }
  }
}

template <int BN, bool A_MN, bool B_MN, int EPI, bool PAIR, bool FB>
__global__ void __launch_bounds__(Cfg<BN, PAIR, EPI, FB>::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmD, const __grid_constant__ CUtensorMap tmD2,
                const __grid_constant__ CUtensorMap tmR, const KArgs p) {
  using C = Cfg<BN, PAIR, EPI, FB>;
  static_assert(!FB || (!A_MN && !B_MN && !C::F32), "fused B: forward GEMMs only");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  uint8_t* panel = smem;  // FB: resident B panel (PANEL_BYTES; 0 otherwise)
  uint8_t* sA = smem + C::PANEL_BYTES;
  uint8_t* sB = sA + C::STAGES * C::A_BYTES;
  uint8_t* staging = sA + C::STAGES * C::STAGE_BYTES;  // 1024-aligned
  uint8_t* rstage = staging + C::STAGING_BYTES;          // R chunks (HAS_R)
  uint64_t* full = reinterpret_cast<uint64_t*>(rstage + C::R_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* mma_done = tempty + 2;
  uint64_t* panel_full = mma_done + 1;  // FB: the panel of the next N block is written
  uint64_t* rbar = panel_full + 1;      // EW epilogue warps x R_BUFS
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(rbar + C::EW * C::R_BUFS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* prod_pos = const_cast<int*>(abort_flag) + 1;  // producer ring position at exit
  int* mma_pos = prod_pos + 1;                        // MMA ring position at exit

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  // Position in the CTA pair (PAIR): rank 0 is the leader that issues the MMAs
  // and owns the full / tmem-empty barriers both CTAs signal.
  const uint32_t rank = PAIR ? cluster_ctarank() : 0u;
  const bool leader = (rank == 0);
  const int unit = PAIR ? static_cast<int>(blockIdx.x >> 1) : static_cast<int>(blockIdx.x);
  const int units = PAIR ? static_cast<int>(gridDim.x >> 1) : static_cast<int>(gridDim.x);
  // Tiles of this CTA (pair): every units-th tile, N block fastest; FB: one
  // contiguous run in N-block-major order, so the B panel changes rarely.
  int t_begin = unit, t_end = p.num_tiles, t_step = units;
  if constexpr (FB) {
    t_begin = static_cast<int>(static_cast<int64_t>(unit) * p.num_tiles / units);
    t_end = static_cast<int>(static_cast<int64_t>(unit + 1) * p.num_tiles / units);
    t_step = 1;
  }
  // FB: within N block nb the M blocks are rotated so that the run starting
  // inside nb (at position base) begins at M block 0.  Every run then walks the
  // M blocks in step with the runs of the other N blocks, and the concurrent
  // pairs read a handful of A tiles (shared through L2) instead of one each.
  auto fb_base = [&](int nb) {
    const int64_t x = static_cast<int64_t>(nb) * p.num_m_blk;
    const int64_t q = (x * units + p.num_tiles - 1) / p.num_tiles;  // first run starting at or after x
    if (q >= units) return 0;
    const int64_t s = q * p.num_tiles / units;
    return s < x + p.num_m_blk ? static_cast<int>(s - x) : 0;
  };
  auto tile_nb = [&](int t) { return FB ? t / p.num_m_blk : t % p.num_n_blk; };
  auto tile_mb = [&](int t) {
    if constexpr (FB) {
      const int nb = t / p.num_m_blk;
      const int r = t - nb * p.num_m_blk - fb_base(nb);
      return r < 0 ? r + p.num_m_blk : r;
    }
    return (t / p.num_n_blk) % p.num_m_blk;
  };
  auto tile_sp = [&](int t) { return FB ? 0 : t / (p.num_n_blk * p.num_m_blk); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], PAIR ? 2 * C::EW : C::EW);
    }
    mbar_init(mma_done, 1);
    mbar_init(panel_full, PAIR ? 2 * C::EW : C::EW);
    for (int i = 0; i < C::EW * C::R_BUFS; ++i) mbar_init(&rbar[i], 1);
    *abort_flag = 0;
    *prod_pos = 0;
    *mma_pos = 0;
    fence_mbar_init();
    tma_prefetch_desc(&tmA);
    if constexpr (!FB) tma_prefetch_desc(&tmB);
    tma_prefetch_desc(&tmD);
    if constexpr (epi_reads_r(EPI)) tma_prefetch_desc(&tmR);
  }
  if (warp == 1) {
    if constexpr (PAIR) {
      tmem_alloc_pair(tmem_slot, C::TMEM_COLS);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(tmem_slot, C::TMEM_COLS);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // Launched as a programmatic dependent of the previous kernel in the stream:
  // everything above (barriers, TMEM, descriptor prefetch) overlapped its tail;
  // no global memory is touched before the previous grid has completed.  Then
  // let the next GEMM's CTAs launch onto SMs as this grid's CTAs retire.
  grid_dependency_wait();
  grid_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer
      int stage = 0, pos = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = t_begin; ok && tile < t_end; tile += t_step) {
        const int nb = tile_nb(tile);
        const int mb = tile_mb(tile);
        const int sp = tile_sp(tile);
        const int kb0 = sp * p.kblk_per_split;
        const int kb1 = min(kb0 + p.kblk_per_split, p.kblk_total);
        const int m0 = mb * C::TILE_M + static_cast<int>(rank) * BM;
        const int n0 = nb * BN + static_cast<int>(rank) * C::B_ROWS;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, abort_flag, p.err)) { ok = false; break; }
          const int k0 = kb * BK;
          uint8_t* a_dst = sA + stage * C::A_BYTES;
          uint8_t* b_dst = sB + stage * C::B_BYTES;
          if constexpr (PAIR) {
            // both CTAs' bytes complete on the leader's full barrier
            const uint32_t bar = mapa_shared(smem_u32(&full[stage]), 0);
            if (leader) mbar_arrive_expect_tx(&full[stage], 2 * C::STAGE_BYTES);
            if constexpr (!A_MN) {
              tma_load_2d_pair(&tmA, bar, a_dst, k0, m0);
            } else {
              tma_load_2d_pair(&tmA, bar, a_dst, m0, k0);
              tma_load_2d_pair(&tmA, bar, a_dst + 64 * 128, m0 + 64, k0);
            }
            if constexpr (FB) {
              // B comes from the resident panel
            } else if constexpr (!B_MN) {
              tma_load_2d_pair(&tmB, bar, b_dst, k0, n0);
            } else {
#pragma unroll
              for (int j = 0; j < C::B_ROWS / 64; ++j)
                tma_load_2d_pair(&tmB, bar, b_dst + j * 64 * 128, n0 + j * 64, k0);
            }
          } else {
            mbar_arrive_expect_tx(&full[stage], C::STAGE_BYTES);
            if constexpr (!A_MN) {
              tma_load_2d(&tmA, &full[stage], a_dst, k0, m0);
            } else {
              tma_load_2d(&tmA, &full[stage], a_dst, m0, k0);
              tma_load_2d(&tmA, &full[stage], a_dst + 64 * 128, m0 + 64, k0);
            }
            if constexpr (FB) {
              // B comes from the resident panel
            } else if constexpr (!B_MN) {
              tma_load_2d(&tmB, &full[stage], b_dst, k0, n0);
            } else {
#pragma unroll
              for (int j = 0; j < C::B_ROWS / 64; ++j)
                tma_load_2d(&tmB, &full[stage], b_dst + j * 64 * 128, n0 + j * 64, k0);
            }
          }
          ++pos;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      *prod_pos = pos;
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      // ------------------------------------------------ MMA issuer
      constexpr uint32_t IDESC = idesc_bf16(C::TILE_M, BN, A_MN, B_MN);
      int stage = 0, pos = 0;
      uint32_t phase = 0;
      int acc = 0;
      uint32_t acc_phase = 0;
      bool ok = true;
      // Arrive on a barrier of this CTA and (PAIR) the same barrier of the peer.
      auto commit_both = [&](uint64_t* bar) {
        if constexpr (PAIR) {
          umma_commit_pair(smem_u32(bar));
          umma_commit_pair(mapa_shared(smem_u32(bar), 1));
        } else {
          umma_commit(bar);
        }
      };
      int panel_nb = -1;  // FB: N block whose panel the MMAs read
      uint32_t panel_phase = 0;
      for (int tile = t_begin; ok && tile < t_end; tile += t_step) {
        const int sp = tile_sp(tile);
        const int kb0 = sp * p.kblk_per_split;
        const int kb1 = min(kb0 + p.kblk_per_split, p.kblk_total);
        if constexpr (FB) {
          if (tile_nb(tile) != panel_nb) {  // both CTAs' epilogue warps wrote the new panel
            if (!mbar_wait(panel_full, panel_phase, abort_flag, p.err)) break;
            panel_phase ^= 1u;
            panel_nb = tile_nb(tile);
            tc_fence_after();
          }
        }
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, abort_flag, p.err)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(acc * BN);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(sA + stage * C::A_BYTES);
          const uint32_t b_base = FB ? smem_u32(panel + kb * C::KB_BYTES)
                                     : smem_u32(sB + stage * C::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = A_MN ? sw128_desc(a_base + kk * 2048, 64 * 128, 1024)
                                     : sw128_desc(a_base + kk * 32, 16, 1024);
            const uint64_t bd = B_MN ? sw128_desc(b_base + kk * 2048, 64 * 128, 1024)
                                     : sw128_desc(b_base + kk * 32, 16, 1024);
            const uint32_t accum = (kb > kb0 || kk > 0) ? 1u : 0u;
            if constexpr (PAIR) umma_bf16_pair(d_tmem, ad, bd, IDESC, accum);
            else umma_bf16(d_tmem, ad, bd, IDESC, accum);
          }
          commit_both(&empty[stage]);
          ++pos;
          if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        commit_both(&tfull[acc]);
        acc ^= 1;
        if (acc == 0) acc_phase ^= 1u;
      }
      // Wait (bounded) for every MMA this thread issued before TMEM is freed.
      if constexpr (PAIR) umma_commit_pair(smem_u32(mma_done)); else umma_commit(mma_done);
      mbar_wait(mma_done, 0, abort_flag, p.err);
      *mma_pos = pos;
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..)
    constexpr bool kF32 = C::F32;
    constexpr bool kR = C::HAS_R;
    constexpr int kSplit = C::EW / 4;  // warps sharing one TMEM lane quarter
    const int q = warp & 3;            // TMEM lane quarter this warp may access
    const int ew = warp - 2;           // epilogue warp index
    const int h = ew >> 2;             // this warp's chunks: h, h + kSplit, ...
    const uint32_t wbuf = smem_u32(staging) + static_cast<uint32_t>(ew * C::WBUF);
    uint8_t* rbuf = rstage + ew * C::R_BUFS * 2048;
    uint64_t* rb = rbar + ew * C::R_BUFS;
    const bool keep_pre = epi_act_fwd(EPI) && p.D != nullptr;
    int acc = 0;
    uint32_t acc_phase = 0;
    uint32_t chunk = 0;
    uint32_t r_issued = 0, r_used = 0;  // R ring: chunks requested / consumed
    // the leader's tmem-empty barrier, which both CTAs' epilogues release
    const uint32_t tempty_leader = PAIR ? mapa_shared(smem_u32(tempty), 0) : smem_u32(tempty);
    // FB: L2 prefetch of this CTA's weight rows of N block nb (one thread).
    auto prefetch_panel = [&](int nb) {
      const int n0 = nb * BN + static_cast<int>(rank) * C::B_ROWS;
      const int rows = min(C::B_ROWS, p.N - n0);
      if (rows <= 0) return;
      const char* src = reinterpret_cast<const char*>(p.W + static_cast<int64_t>(n0) * p.K);
      int64_t bytes = static_cast<int64_t>(rows) * p.K * 4;
      for (; bytes > 0; bytes -= 65536, src += 65536)
        bulk_prefetch_l2(src, static_cast<uint32_t>(bytes < 65536 ? bytes : 65536));
    };
    // FB: write the panel of N block nb (this CTA's B_ROWS rows) and tell the MMA.
    auto produce_panel = [&](int nb) {
      if constexpr (FB) {
        const int n_base = nb * BN + static_cast<int>(rank) * C::B_ROWS;
        if (p.bits == 6) convert_panel<C, 6>(p, panel, n_base, ew, lane);
        else if (p.bits == 5) convert_panel<C, 5>(p, panel, n_base, ew, lane);
        else convert_panel<C, 8>(p, panel, n_base, ew, lane);
        fence_proxy_async_smem();  // generic-proxy writes visible to the tensor cores
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR) mbar_arrive_cluster(mapa_shared(smem_u32(panel_full), 0));
          else mbar_arrive(panel_full);
        }
      }
    };
    if constexpr (FB) {
      if (ew == 0 && lane == 0) {
        // L2 prefetch of the weight rows of the first few panels this CTA converts
        int last = -1, count = 0;
        for (int t = t_begin; t < t_end && count < 4; ++t) {
          const int nb = tile_nb(t);
          if (nb == last) continue;
          last = nb;
          ++count;
          prefetch_panel(nb);
        }
      }
      if (t_begin < t_end) produce_panel(tile_nb(t_begin));
    }
    for (int tile = t_begin; tile < t_end; tile += t_step) {
      const int nb = tile_nb(tile);
      const int mb = tile_mb(tile);
      if constexpr (FB) {
        // refresh the L2 copy of the next panel's rows a few tiles before it is
        // built (the start-of-kernel prefetch is long evicted by then)
        constexpr int kAhead = 3;
        if (ew == 0 && lane == 0 && tile + kAhead < t_end &&
            tile_nb(tile + kAhead) != tile_nb(tile + kAhead - 1))
          prefetch_panel(tile_nb(tile + kAhead));
      }
      const int row0 = mb * C::TILE_M + static_cast<int>(rank) * BM + q * 32;
      const int ncols = min(BN, p.N - nb * BN);
      const int nchunks = (ncols + 31) / 32;
      const int mine = nchunks > h ? (nchunks - h + kSplit - 1) / kSplit : 0;
      // Request this warp's first R chunks before waiting for the accumulator.
      auto issue_r = [&](int i) {
        if (lane == 0) {
          const uint32_t slot = r_issued % C::R_BUFS;
          mbar_arrive_expect_tx(&rb[slot], 2048);
          tma_load_2d(&tmR, &rb[slot], rbuf + slot * 2048, nb * BN + (h + i * kSplit) * 32, row0);
        }
        ++r_issued;
      };
      if constexpr (kR) {
        for (int i = 0; i < mine && i < C::R_BUFS; ++i) issue_r(i);
      }
      if (!mbar_wait(&tfull[acc], acc_phase, abort_flag, p.err)) break;
      tc_fence_after();
      if constexpr (FB) {
        // Every MMA of this tile has completed, so the old panel is free: write
        // the next N block's panel first (the MMA waits on it), then drain this
        // tile's accumulator while the next tile runs.
        if (tile + 1 < t_end && tile_nb(tile + 1) != nb) produce_panel(tile_nb(tile + 1));
      }
      const uint32_t t_row = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(acc * BN);
      auto release_acc = [&]() {  // this warp's part of the accumulator is read
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if constexpr (PAIR) mbar_arrive_cluster(tempty_leader + 8u * static_cast<uint32_t>(acc));
          else mbar_arrive(&tempty[acc]);
        }
      };
      if (mine == 0) release_acc();
      bool ok = true;
#pragma unroll 1
      for (int i = 0; i < mine; ++i, ++chunk) {
        const int c = h + i * kSplit;
        const int col0 = nb * BN + c * 32;
        uint4 rin[4] = {};
        if constexpr (kR) {
          const uint32_t slot = r_used % C::R_BUFS;
          if (!mbar_wait(&rb[slot], (r_used / C::R_BUFS) & 1u, abort_flag, p.err)) { ok = false; break; }
          const uint32_t base = smem_u32(rbuf + slot * 2048) + static_cast<uint32_t>(lane) * 64u;
          const int sw = (lane >> 1) & 3;
#pragma unroll
          for (int g = 0; g < 4; ++g) rin[g] = ld_shared_v4(base + (static_cast<uint32_t>(g ^ sw) << 4));
          ++r_used;
          fence_proxy_async_smem();  // reads done before the slot is refilled by TMA
          __syncwarp();
          if (i + C::R_BUFS < mine) issue_r(i + C::R_BUFS);
        }
        uint32_t r[32];
        tmem_ld32(t_row + static_cast<uint32_t>(c * 32), r);
        tmem_ld_wait();
        if (i == mine - 1) release_acc();  // hand the accumulator back to the MMA
        const uint32_t b = chunk & 1u;
        const uint32_t buf0 = kF32 ? wbuf + b * 4096u : wbuf + b * 2048u;
        const uint32_t buf1 = wbuf + 4096u + b * 2048u;
        if (lane == 0) bulk_wait_read<1>();  // the store that last used buffer b is done reading
        __syncwarp();
        stage_chunk<EPI>(p, r, rin, buf0, buf1, lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          const uint8_t* s0 = staging + (buf0 - smem_u32(staging));
          if constexpr (EPI == EPI_F32_ATOMIC) {
            tma_reduce_add_2d(&tmD, s0, col0, row0);
          } else if constexpr (epi_act_fwd(EPI)) {
            if (keep_pre) tma_store_2d(&tmD, s0, col0, row0);
            tma_store_2d(&tmD2, staging + (buf1 - smem_u32(staging)), col0, row0);
          } else {
            tma_store_2d(&tmD, s0, col0, row0);
          }
          bulk_commit();
        }
      }
      if (!ok) break;
      acc ^= 1;
      if (acc == 0) acc_phase ^= 1u;
    }
    // R chunks requested but not consumed (only after a timeout): let them land.
    if (kR && lane == 0) {
      for (uint32_t k = r_used; k < r_issued; ++k)
        mbar_drain(&rb[k % C::R_BUFS], (k / C::R_BUFS) & 1u);
    }
    if (lane == 0) bulk_wait_all();  // every output chunk written before the block exits
    __syncwarp();
  }

  __syncthreads();
  if (threadIdx.x == 0 && *abort_flag) {
    // Drain: wait (bounded) for tiles the producer requested but the MMA never
    // consumed, so no TMA write lands after the block exits.
    int stage = *mma_pos % C::STAGES;
    uint32_t phase = static_cast<uint32_t>((*mma_pos / C::STAGES) & 1);
    const unsigned long long t0 = globaltimer_ns();
    for (int i = *mma_pos; i < *prod_pos; ++i) {
      while (!mbar_try_wait(&full[stage], phase))
        if (globaltimer_ns() - t0 > kWaitLimitNs) break;
      if (++stage == C::STAGES) { stage = 0; phase ^= 1u; }
    }
  }
  // No CTA of a pair leaves while its peer may still signal its barriers.
  if constexpr (PAIR) cluster_sync(); else __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    if constexpr (PAIR) tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
    else tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode() {
  static EncodeFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeFn>(f);
  });
  return fn;
}

// 2-D bf16 tensor map: inner dimension `inner` (contiguous), outer `outer`,
// row stride `ld` elements, box {64, box_outer}, 128-byte swizzle.
int make_map(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t ld,
             int box_outer) {
  EncodeFn enc = get_encode();
  if (!enc) return QAT_ERR_UNSUPPORTED;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_outer)};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? QAT_OK : QAT_ERR_ARG;
}

// Output tensor map: inner dimension `inner` (N), outer `outer` (M), row stride
// `ld` elements, box 32 x 32, bf16 (64-byte swizzle) or fp32 (128-byte swizzle).
int make_out_map(CUtensorMap* m, const void* base, int64_t inner, int64_t outer, int64_t ld,
                 bool f32) {
  EncodeFn enc = get_encode();
  if (!enc) return QAT_ERR_UNSUPPORTED;
  const int eb = f32 ? 4 : 2;
  cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(outer)};
  cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * eb};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                   const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   f32 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? QAT_OK : QAT_ERR_ARG;
}

template <int BN, bool A_MN, bool B_MN, int EPI, bool PAIR, bool FB = false>
int launch_t(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& md,
             const CUtensorMap& md2, const CUtensorMap& mr, const KArgs& a, cudaStream_t s) {
  using C = Cfg<BN, PAIR, EPI, FB>;
  auto kern = gemm_kernel<BN, A_MN, B_MN, EPI, PAIR, FB>;
  // the shared-memory attribute belongs to each device's context: set it once
  // per instantiation and device, before the first launch there
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  if (!device_flag_once(attr_done, &dev)) {
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
    if (e != cudaSuccess) return QAT_ERR_CUDA;
    device_flag_set(attr_done, dev);
  }
  const int units = PAIR ? sm_count() / 2 : sm_count();
  const int grid = std::max(1, std::min(a.num_tiles, units)) * (PAIR ? 2 : 1);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(C::THREADS);
  cfg.dynamicSmemBytes = C::SMEM_BYTES;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = PAIR ? 2 : 1;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // programmatic dependent launch (the kernel waits with griddepcontrol.wait)
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ma, mb, md, md2, mr, a);
  count_launch();
  return cuda_status(e == cudaSuccess ? cudaGetLastError() : e);
}

template <int BN, bool PAIR>
int dispatch_bn(const GemmDesc& g, const CUtensorMap& ma, const CUtensorMap& mb,
                const CUtensorMap& md, const CUtensorMap& md2, const CUtensorMap& mr,
                const KArgs& a, int epi, cudaStream_t s) {
  if (!g.a_mn && !g.b_mn) {
    switch (epi) {
      case EPI_BF16: return launch_t<BN, false, false, EPI_BF16, PAIR>(ma, mb, md, md2, mr, a, s);
      case EPI_BF16_RESID:
        return launch_t<BN, false, false, EPI_BF16_RESID, PAIR>(ma, mb, md, md2, mr, a, s);
      case EPI_RELU2: return launch_t<BN, false, false, EPI_RELU2, PAIR>(ma, mb, md, md2, mr, a, s);
      case EPI_LRELU2:
        return launch_t<BN, false, false, EPI_LRELU2, PAIR>(ma, mb, md, md2, mr, a, s);
      default: break;
    }
  } else if (!g.a_mn && g.b_mn) {
    switch (epi) {
      case EPI_BF16: return launch_t<BN, false, true, EPI_BF16, PAIR>(ma, mb, md, md2, mr, a, s);
      case EPI_BF16_RESID:
        return launch_t<BN, false, true, EPI_BF16_RESID, PAIR>(ma, mb, md, md2, mr, a, s);
      case EPI_DRELU2: return launch_t<BN, false, true, EPI_DRELU2, PAIR>(ma, mb, md, md2, mr, a, s);
      case EPI_DLRELU2:
        return launch_t<BN, false, true, EPI_DLRELU2, PAIR>(ma, mb, md, md2, mr, a, s);
      default: break;
    }
  } else if (g.a_mn && g.b_mn) {
    switch (epi) {
      case EPI_F32: return launch_t<BN, true, true, EPI_F32, PAIR>(ma, mb, md, md2, mr, a, s);
      case EPI_F32_ATOMIC:
        return launch_t<BN, true, true, EPI_F32_ATOMIC, PAIR>(ma, mb, md, md2, mr, a, s);
      default: break;
    }
  }
  return QAT_ERR_ARG;  // combination not instantiated
}

// Fused-B forward GEMMs (paired CTAs, K-major operands).
template <int BN>
int dispatch_fb(const CUtensorMap& ma, const CUtensorMap& md, const CUtensorMap& md2,
                const CUtensorMap& mr, const KArgs& a, int epi, cudaStream_t s) {
  switch (epi) {
    case EPI_BF16: return launch_t<BN, false, false, EPI_BF16, true, true>(ma, ma, md, md2, mr, a, s);
    case EPI_BF16_RESID:
      return launch_t<BN, false, false, EPI_BF16_RESID, true, true>(ma, ma, md, md2, mr, a, s);
    case EPI_RELU2: return launch_t<BN, false, false, EPI_RELU2, true, true>(ma, ma, md, md2, mr, a, s);
    case EPI_LRELU2:
      return launch_t<BN, false, false, EPI_LRELU2, true, true>(ma, ma, md, md2, mr, a, s);
    default: return QAT_ERR_ARG;
  }
}

// N tile of the fused-B GEMM: the panel (BN/2 rows x K bf16 per CTA) must fit
// its KBP k-blocks; widest tile that divides N first.  0 = not supported.
int fused_b_bn(int64_t N, int64_t K) {
  const int64_t kblk = (K + BK - 1) / BK;
  const bool k256 = kblk <= Cfg<256, true, EPI_BF16, true>::KBP;
  const bool k192 = kblk <= Cfg<192, true, EPI_BF16, true>::KBP;
  const bool k160 = kblk <= Cfg<160, true, EPI_BF16, true>::KBP;
  const bool k128 = kblk <= Cfg<128, true, EPI_BF16, true>::KBP;
  if (k256 && N % 256 == 0) return 256;
  if (k192 && N % 192 == 0) return 192;
  if (k160 && N % 160 == 0) return 160;
  if (k256) return 256;
  if (k128) return 128;
  return 0;
}

// Split count for the fp32 weight-gradient GEMMs: minimise the makespan
// ceil(tiles*s / SMs) * (ceil(kblk / s) + E), preferring fewer splits, where
// E = kSplitCost k-blocks charges each split work unit for its partial tile's
// fp32 reduce-add and the zero-fill.  (Measured, 16 against 0, 28 and 48: the
// MLP's 512 x 2048 weight gradients at 65,536 tokens 109 -> 103 us -- 9 splits
// instead of 32 -- and the d = 640 core's training step 1.106 -> 1.064 ms.)
constexpr int kSplitCost = 16;
int choose_splits(int tiles, int kblk, int sms) {
  int best_s = 1;
  long long best = -1;
  for (int s = 1; s <= std::min(kblk, 64); ++s) {
    const long long waves = (static_cast<long long>(tiles) * s + sms - 1) / sms;
    const long long cost = waves * ((kblk + s - 1) / s + (s > 1 ? kSplitCost : 0));
    if (best < 0 || cost < best) {
      best = cost;
      best_s = s;
    }
  }
  return best_s;
}

}  // namespace

bool fused_b_supported(int64_t M, int64_t N, int64_t K, int epi) {
  const bool fwd_epi = epi == EPI_BF16 || epi == EPI_BF16_RESID || epi == EPI_RELU2 || epi == EPI_LRELU2;
  return fwd_epi && M >= 256 && N > 0 && K > 0 && (K & 7) == 0 && fused_b_bn(N, K) != 0;
}

int launch_gemm(const GemmDesc& g, cudaStream_t stream) {
  if (g.M < 0 || g.N <= 0 || g.K <= 0) return QAT_ERR_ARG;
  if (g.M == 0) return QAT_OK;
  if (!g.A || (!g.B && !g.Wraw) || (!g.D && !epi_act_fwd(g.epi))) return QAT_ERR_ARG;
  if (g.Wraw && (!fused_b_supported(g.M, g.N, g.K, g.epi) || g.a_mn || g.b_mn))
    return QAT_ERR_UNSUPPORTED;
  if (g.Wraw && (!aligned16(g.Wraw) || (g.bits != 5 && g.bits != 6 && g.bits != 8)))
    return g.bits == 5 || g.bits == 6 || g.bits == 8 ? QAT_ERR_ALIGN : QAT_ERR_ARG;
  if (epi_act_fwd(g.epi) && !g.D2) return QAT_ERR_ARG;
  if (epi_reads_r(g.epi) && !g.R) return QAT_ERR_ARG;
  if (!aligned16(g.A) || (g.B && !aligned16(g.B)) || (g.D && !aligned16(g.D)) || (g.D2 && !aligned16(g.D2)) ||
      (g.R && !aligned16(g.R)))
    return QAT_ERR_ALIGN;
  if ((g.N & 7) || (g.lda & 7) || (g.ldb & 7) || (g.ldd & 7) || (g.D2 && (g.ldd2 & 7)) ||
      (g.R && (g.ldr & 7)))
    return QAT_ERR_SHAPE;
  if (g.M > (1ll << 31) - 256 || g.N > (1 << 30) || g.K > (1ll << 31) - 256) return QAT_ERR_SHAPE;

  // N tile.  GEMMs with at least 256 rows run on CTA pairs 256 columns wide,
  // the last N block partial where 256 does not divide N: the forward and dX
  // GEMMs (bf16 output) when N >= 160, and the weight-gradient GEMMs (both
  // operands MN-major).  The rest take 256 (paired when M >= 256) unless 128
  // wastes fewer columns.  (For the d = 640 core's backward, 256-wide pairs
  // against 128-wide single-CTA tiles: dX GEMMs 57 -> 44 us (N = 640,
  // K = 1920) and 58 -> 50 us (N = 1920, K = 640), weight gradients 33 -> 25 us
  // (640 x 640) and 70 -> 64 us (1920 x 640), per 16,384 tokens.)
  int BN;
  bool pair;
  const bool kmajor_fwd = (!g.a_mn && g.epi != EPI_F32 && g.epi != EPI_F32_ATOMIC) ||
                          (g.a_mn && g.M >= 256);
  if (g.Wraw) {
    pair = true;
    BN = fused_b_bn(g.N, g.K);
  } else if (kmajor_fwd && g.M >= 256 && g.N >= 160) {
    pair = true;
    // (a wave-count rule -- the width of fewest ceil(tiles / pairs) * BN -- was
    // slower: 160-wide tiles for the d = 640 core's N = 1280 filled the waves
    // better but cost more operand traffic per FLOP, core 0.42 -> 0.44 ms)
    // 256 wide even when it does not divide N (the last N block is partial):
    // narrower tiles re-read A once more per FLOP, and with K this short the
    // operand stream from L2 then sets the pace (d = 640 core: 160-wide tiles
    // for N = 640, 192-wide for N = 1920 took 0.417 ms per R = 3 forward,
    // 256-wide everywhere 0.365 ms)
    BN = 256;
  } else {
    const int64_t pad256 = (g.N + 255) / 256 * 256 - g.N;
    const int64_t pad128 = (g.N + 127) / 128 * 128 - g.N;
    BN = (pad128 < pad256) ? 128 : 256;
    pair = (BN == 256) && g.M >= 256;
  }
  const int tile_m = pair ? 2 * BM : BM;

  KArgs a{};
  a.M = static_cast<int>(g.M);
  a.N = static_cast<int>(g.N);
  a.num_m_blk = static_cast<int>((g.M + tile_m - 1) / tile_m);
  a.num_n_blk = static_cast<int>((g.N + BN - 1) / BN);
  a.kblk_total = static_cast<int>((g.K + BK - 1) / BK);
  a.splits = 1;
  a.D = g.D;
  a.ldd = g.ldd;
  a.D2 = g.D2;
  a.ldd2 = g.ldd2;
  a.R = reinterpret_cast<const __nv_bfloat16*>(g.R);
  a.ldr = g.ldr;
  a.accumulate = g.accumulate ? 1 : 0;
  a.err = device_error_ptr();
  a.W = g.Wraw;
  a.K = static_cast<int>(g.K);
  a.bits = g.bits;

  int epi = g.epi;
  if (epi == EPI_F32 || epi == EPI_F32_ATOMIC) {
    const int tiles = a.num_m_blk * a.num_n_blk;
    // Split K only while the output tiles occupy fewer than half the CTAs
    // (pairs): with more tiles, a wave of whole tiles already keeps at least
    // half of them busy, and the split's zero-fill and fp32 reduce-adds cost
    // more than the better wave fill returns (head dW 8192 x 512 over 65,536
    // tokens: 64 tiles on 74 pairs, 447-461 us split 8 ways, 424-426 us whole).
    const int cunits = pair ? sm_count() / 2 : sm_count();
    int s = (2 * tiles >= cunits) ? 1 : choose_splits(tiles, a.kblk_total, cunits);
    a.kblk_per_split = (a.kblk_total + s - 1) / s;
    s = (a.kblk_total + a.kblk_per_split - 1) / a.kblk_per_split;  // no empty split
    a.splits = s;
    if (s > 1 || g.accumulate) {
      if (!g.accumulate) {
        cudaError_t e = (g.ldd == g.N)
                            ? cudaMemsetAsync(g.D, 0, static_cast<size_t>(g.M * g.N) * 4, stream)
                            : cudaMemset2DAsync(g.D, static_cast<size_t>(g.ldd) * 4, 0,
                                                static_cast<size_t>(g.N) * 4,
                                                static_cast<size_t>(g.M), stream);
        if (e != cudaSuccess) return QAT_ERR_CUDA;
      }
      epi = EPI_F32_ATOMIC;
    } else {
      epi = EPI_F32;
    }
  } else {
    a.kblk_per_split = a.kblk_total;
  }
  const int64_t tiles64 = static_cast<int64_t>(a.num_m_blk) * a.num_n_blk * a.splits;
  if (tiles64 > (1ll << 31) - 1) return QAT_ERR_SHAPE;
  a.num_tiles = static_cast<int>(tiles64);

  CUtensorMap ma, mb;
  const int b_rows = pair ? BN / 2 : BN;  // B rows one CTA stages
  int rc = g.a_mn ? make_map(&ma, g.A, g.M, g.K, g.lda, 64)
                  : make_map(&ma, g.A, g.K, g.M, g.lda, BM);
  if (rc) return rc;
  if (g.Wraw) {
    mb = ma;  // unused: B is quantized from Wraw inside the kernel
  } else {
    rc = g.b_mn ? make_map(&mb, g.B, g.N, g.K, g.ldb, 64)
                : make_map(&mb, g.B, g.K, g.N, g.ldb, b_rows);
    if (rc) return rc;
  }
  // Output maps: 32x32 boxes, bf16 with 64-byte swizzle or fp32 with 128-byte swizzle.
  CUtensorMap md, md2;
  const bool f32 = (epi == EPI_F32 || epi == EPI_F32_ATOMIC);
  const void* d_base = g.D ? g.D : g.D2;
  const int64_t d_ld = g.D ? g.ldd : g.ldd2;
  rc = make_out_map(&md, d_base, g.N, g.M, d_ld, f32);
  if (rc) return rc;
  rc = make_out_map(&md2, g.D2 ? g.D2 : d_base, g.N, g.M, g.D2 ? g.ldd2 : d_ld, false);
  if (rc) return rc;
  CUtensorMap mr = md;
  if (epi_reads_r(g.epi)) {
    rc = make_out_map(&mr, g.R, g.N, g.M, g.ldr, false);
    if (rc) return rc;
  }
  if (g.Wraw) {
    switch (BN) {
      case 128: return dispatch_fb<128>(ma, md, md2, mr, a, epi, stream);
      case 160: return dispatch_fb<160>(ma, md, md2, mr, a, epi, stream);
      case 192: return dispatch_fb<192>(ma, md, md2, mr, a, epi, stream);
      default: return dispatch_fb<256>(ma, md, md2, mr, a, epi, stream);
    }
  }
  if (pair) return dispatch_bn<256, true>(g, ma, mb, md, md2, mr, a, epi, stream);
  return BN == 256 ? dispatch_bn<256, false>(g, ma, mb, md, md2, mr, a, epi, stream)
                   : dispatch_bn<128, false>(g, ma, mb, md, md2, mr, a, epi, stream);
}

}  // namespace qat
