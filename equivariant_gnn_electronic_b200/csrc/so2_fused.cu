// Fused eSCN layer on tcgen05: SO(2) linear, attention, rotate-back and aggregation in
// one kernel per range of edge tiles, so that neither the per-edge SO(2) outputs y nor
// the messages msg_e are ever stored.
//
// Method: "MALOQ: Massively Accelerated Learning of Operators for Quantum Transport",
// Sections II-B1 and III (rotate each edge onto one axis, SO(2) constrained linear
// layers, aggregate onto the target node) and Section III-D / Fig. 4(b) (message from
// the concatenated pair); incoming-edge ownership, attention and aggregation local to
// the owner of the edges: review page of "Distributed Equivariant Graph Neural
// Networks for Large-Scale Electronic Structure Prediction", "What carries the
// argument".
//
// Orientation.  The SO(2) linear runs with the weights as the MMA's M operand and the
// edges as N: D[128 output channels][128 edges] += W[128 x K] X[128 edges x K]^T, so a
// TMEM lane holds one output channel c of one (degree l, order m) row for the 128
// edges of a tile.  Each epilogue thread owns one channel c (four warps, one per TMEM
// lane quadrant, C = 128) and sums over edges in registers: the rotate-back
// msg_e[l, m', c] = sum_m D^l_e[m, m'] y_e[l, m, c] and the weighted segment sum over
// each destination atom's edges need no data from other threads.
//
// Per 128-edge tile the passes run |m| = 0 first (two degrees per pass), then the
// (+m, -m) pairs (one degree per pass: y+ in TMEM columns 0-127, y- in 128-255; four
// MMAs per K step, one with the negate-A bit).  Epilogue:
//   |m| = 0 passes: y0 goes to a per-CTA stash in bf16 (it cannot be aggregated before
//     the attention weights exist) and SiLU(y0) feeds the logits a_e = A SiLU(y0_e)
//     + bA through warp-level mma.sync on 16 x 16 blocks (the logits reduce over
//     channels, i.e. across threads);
//   softmax statistics per head over each destination's edges inside the tile
//     (maximum, sum of exp), p_e = exp(a_e - max);
//   y0 from the stash and then each (+m, -m) pass: acc[m'] += p_e D^l_e[m, m'] y_e,
//     flushed at each destination change into that destination's record;
//   end of tile: destinations whose edges all lie in the tile are finished here,
//     out_d = n_d + acc / sum; destinations whose edges cross a tile boundary leave a
//     partial record (acc, max, sum) per tile, merged by combine_kernel.
// No atomics between threads: every accumulator element has one writing thread.
#include <math.h>

#include "common.cuh"
#include "so2_tc.cuh"
#include "tc_ptx.cuh"

namespace {

constexpr int kMaxXS = 8;           // x tile stages (128 edges x 64 K, bf16, 16 KB): 3..8 per launch
constexpr int kMaxWS = 3;           // weight tile stages (<= 256 rows x 64 K, bf16, 32 KB): 2..3 per launch
constexpr int kXBytes = 128 * 128;
constexpr int kWBytes = 256 * 128;
constexpr int kFThreads = 10 * 32;  // warp 0 bulk copies, warp 1 MMA, warps 2-9 epilogue
constexpr uint32_t kEpiBar = 1;     // named barrier of the 256 epilogue threads

struct FusedCtl {
  uint64_t x_full[kMaxXS], x_empty[kMaxXS], w_full[kMaxWS], w_empty[kMaxWS];
  uint64_t acc_full[2], acc_empty[2], mma_done;
  uint32_t tmem_base;
  int abort;
};

// Epilogue shared memory (after the operand stages).
// The epilogue's work buffer dbuf (sized per launch, after EpiSmem) holds, in turn: the
// partial logits of group 0's warps and their SiLU(y0) staging tiles (|m| = 0 passes),
// the rows m = 0 of every D^l (y0 step), and per group the Wigner rows of its passes.
struct EpiSmem {
  float pw[128 * 16];             // logits a[e][h], then softmax numerators p[e][h]
  float segS[128 * 16];           // softmax denominator of each tile segment and head
  float segM[2 * 16];             // softmax maximum of the two partial (slot) segments
  int dst[128];                   // destination atom of each edge of the tile
  int seg_d[129], seg_b[129], seg_slot[129];
  int wcnt[4];
  int nseg;
};

__device__ __forceinline__ void epi_bar() { tc::bar_sync(kEpiBar, 256); }
__device__ __forceinline__ void group_bar(int g) { tc::bar_sync(2 + g, 128); }

// What the epilogue helpers need of the launch parameters, passed by value (registers)
// rather than as a reference to the kernel's parameter block.
struct EpiArgs {
  float* slots;
  float* acc_g;
  int C, L2, rec_floats;
};

__device__ __forceinline__ float* seg_target(const EpiArgs& A, const EpiSmem* es, int t, int k) {
  const int slot = es->seg_slot[k];
  return slot >= 0 ? A.slots + ((size_t)t * 2 + slot) * A.rec_floats
                   : A.acc_g + (size_t)es->seg_d[k] * A.L2 * A.C;
}

__device__ __forceinline__ int pad4(int x) { return (x + 3) & ~3; }

// acc[m'/2] (pairs of m') += D[m'] * x for m' < NL, D four-float aligned in shared memory.
template <int NL>
__device__ __forceinline__ void axpy_row(float2* acc, const float* D, float x) {
  constexpr int NP = (NL + 3) & ~3;
  const float2 x2 = make_float2(x, x);
  const float4* d4 = reinterpret_cast<const float4*>(D);
#pragma unroll
  for (int u = 0; u < NP / 4; ++u) {
    const float4 w = d4[u];
    if (2 * u < (NL + 1) / 2) acc[2 * u] = __ffma2_rn(make_float2(w.x, w.y), x2, acc[2 * u]);
    if (2 * u + 1 < (NL + 1) / 2) acc[2 * u + 1] = __ffma2_rn(make_float2(w.z, w.w), x2, acc[2 * u + 1]);
  }
}

// Writes (store, first contribution) or adds one segment's sums into its record.
template <int NL, bool ADD>
__device__ __forceinline__ void flush(float* tg, int C, float2* acc) {
#pragma unroll
  for (int m = 0; m < NL; ++m) {
    const float v = (m & 1) ? acc[m >> 1].y : acc[m >> 1].x;
    if (ADD) tc::red_add(tg + (size_t)m * C, v);
    else tg[(size_t)m * C] = v;
  }
#pragma unroll
  for (int i = 0; i < (NL + 1) / 2; ++i) acc[i] = make_float2(0.f, 0.f);
}

// y0 of degree l (NL = 2l + 1) from the stash: for each destination segment k of the
// tile, acc[m'] = sum_e p_e D^l_e[0, m'] y0_e[l, c], stored (first contribution to the
// segment's record).  The thread's stash row holds its channel's 128 edges
// contiguously (bf16), read 32 edges at a time with the next 32 in flight.
template <int NL>
__device__ __noinline__ void y0_degree(const EpiArgs A, const EpiSmem* es, const float* m0r, int t, int l, int c, int hh,
                                       int nvalid, int DZ, int offz, const uint4* st_row) {
  float2 acc[(NL + 1) / 2];
#pragma unroll
  for (int i = 0; i < (NL + 1) / 2; ++i) acc[i] = make_float2(0.f, 0.f);
  int k = 0, nb = es->seg_b[1];
  const int C = A.C;
  const size_t roff = (size_t)(l * l) * C + c;
  uint4 cur[4], nxt[4];
#pragma unroll
  for (int u = 0; u < 4; ++u) cur[u] = st_row[u];
#pragma unroll 1
  for (int j = 0; j < nvalid; j += 32) {
    if (j + 32 < nvalid) {
#pragma unroll
      for (int u = 0; u < 4; ++u) nxt[u] = st_row[(j + 32) / 8 + u];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int j8 = j + 8 * u;
      if (j8 >= nvalid) break;
      float v[8];
      tc::unpack8(cur[u], v);
      if (j8 + 8 <= nb && j8 + 8 <= nvalid) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
          axpy_row<NL>(acc, m0r + (j8 + i) * DZ + offz, es->pw[(j8 + i) * 16 + hh] * v[i]);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int e = j8 + i;
          if (e >= nvalid) break;
          if (e == nb) {
            flush<NL, false>(seg_target(A, es, t, k) + roff, C, acc);
            ++k;
            nb = es->seg_b[k + 1];
          }
          axpy_row<NL>(acc, m0r + e * DZ + offz, es->pw[e * 16 + hh] * v[i]);
        }
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) cur[u] = nxt[u];
  }
  flush<NL, false>(seg_target(A, es, t, k) + roff, C, acc);
}

// 8 edges of a (+b, -b) pass: acc[m'] += p_e (D^l_e[+b, m'] y+_e + D^l_e[-b, m'] y-_e).
// The Wigner rows of the pass are dw[e][2][NP] (shared memory).
template <int NL>
__device__ __forceinline__ void pm_edges(const EpiSmem* es, const float* dw, int hh, int j, int nvalid,
                                         const uint32_t* y, float2* acc, int& k, int& nb, const EpiArgs& A,
                                         int t, size_t roff) {
  constexpr int NP = (NL + 3) & ~3;
  if (j + 8 <= nb && j + 8 <= nvalid) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float pe = es->pw[(j + i) * 16 + hh];
      const float* d = dw + (j + i) * 2 * NP;
      axpy_row<NL>(acc, d, pe * __uint_as_float(y[i]));
      axpy_row<NL>(acc, d + NP, pe * __uint_as_float(y[8 + i]));
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int e = j + i;
    if (e >= nvalid) break;
    if (e == nb) {
      flush<NL, true>(seg_target(A, es, t, k) + roff, A.C, acc);
      ++k;
      nb = es->seg_b[k + 1];
    }
    const float pe = es->pw[e * 16 + hh];
    const float* d = dw + e * 2 * NP;
    axpy_row<NL>(acc, d, pe * __uint_as_float(y[i]));
    axpy_row<NL>(acc, d + NP, pe * __uint_as_float(y[8 + i]));
  }
}

// One (+b, -b) pass of degree l: y+ in TMEM columns [tb, tb + 128), y- in [tb + 128,
// tb + 256), read 8 edges at a time with the next 8 in flight; sums added into each
// destination segment's record.
template <int NL>
__device__ __noinline__ void pm_degree(const EpiArgs A, const EpiSmem* es, const float* dw, int t, int l, int c,
                                       int hh, int nvalid, uint32_t tb) {
  float2 acc[(NL + 1) / 2];
#pragma unroll
  for (int i = 0; i < (NL + 1) / 2; ++i) acc[i] = make_float2(0.f, 0.f);
  int k = 0, nb = es->seg_b[1];
  const size_t roff = (size_t)(l * l) * A.C + c;
  uint32_t ya[16], yb[16];   // [0, 8) y+, [8, 16) y- of 8 edges
  tc::tmem_ld8_issue(tb, ya);
  tc::tmem_ld8_issue(tb + 128, ya + 8);
  tc::tmem_ld_wait8x2(ya, ya + 8);
#pragma unroll 1
  for (int j = 0; j < nvalid; j += 16) {
    const bool more1 = j + 8 < nvalid, more2 = j + 16 < nvalid;
    if (more1) {
      tc::tmem_ld8_issue(tb + j + 8, yb);
      tc::tmem_ld8_issue(tb + 128 + j + 8, yb + 8);
    }
    pm_edges<NL>(es, dw, hh, j, nvalid, ya, acc, k, nb, A, t, roff);
    if (!more1) break;
    tc::tmem_ld_wait8x2(yb, yb + 8);
    if (more2) {
      tc::tmem_ld8_issue(tb + j + 16, ya);
      tc::tmem_ld8_issue(tb + 128 + j + 16, ya + 8);
    }
    pm_edges<NL>(es, dw, hh, j + 8, nvalid, yb, acc, k, nb, A, t, roff);
    if (!more2) break;
    tc::tmem_ld_wait8x2(ya, ya + 8);
  }
  flush<NL, true>(seg_target(A, es, t, k) + roff, A.C, acc);
}

__device__ __forceinline__ bool own_deg(const TcParams& P, int g, int l) { return ((P.own_b >> l) & 1) == g; }
__device__ __forceinline__ int pass_l(const TcParams& P, int p) { return P.pass[p].block + P.pass[p].n_off / 128; }
// The next pass after p whose degree group g owns (P.npass if none).
__device__ __forceinline__ int next_own(const TcParams& P, int g, int p) {
  int r = p + 1;
  while (r < P.npass && !own_deg(P, g, pass_l(P, r))) ++r;
  return r;
}

// Rows (l, +b) and (l, -b) of D^l for edge `ee` of the tile, fetched asynchronously
// (no registers held) into dst[ee][2][pad4(2l + 1)].
__device__ __forceinline__ void fetch_rows(const TcParams& P, int pp, float* dst, int ee, int nvalid, long long e0) {
  const int b2 = P.pass[pp].block, l2 = pass_l(P, pp), dl2 = 2 * l2 + 1, np2 = pad4(dl2);
  const int ml2 = l2 < P.mmax ? l2 : P.mmax;
  if (ee < nvalid) {
    const float* wr = P.wig + (size_t)(e0 + ee) * P.wfl + P.woff[l2];
    const uint32_t dd = tc::smem_u32(dst + ee * 2 * np2);
    for (int m = 0; m < dl2; ++m) {
      tc::cp_async4(dd + 4 * m, wr + (ml2 + b2) * dl2 + m);
      tc::cp_async4(dd + 4 * (np2 + m), wr + (ml2 - b2) * dl2 + m);
    }
  }
}

// |m| = 0 row block of degree l (TMEM columns [tb, tb + 128), thread = channel c):
// y0 into the thread's stash row (the 128 edges contiguous, bf16).
__device__ __noinline__ void m0_stash(uint32_t tb, __nv_bfloat16* row) {
#pragma unroll 1
  for (int j = 0; j < 4; ++j) {
    uint32_t y[32];
    tc::tmem_ld32_issue(tb + 32 * j, y);
    tc::tmem_ld_wait(y);
    uint4* sp = reinterpret_cast<uint4*>(row + 32 * j);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      uint4 w;
      w.x = tc::pack2(__uint_as_float(y[8 * u]), __uint_as_float(y[8 * u + 1]));
      w.y = tc::pack2(__uint_as_float(y[8 * u + 2]), __uint_as_float(y[8 * u + 3]));
      w.z = tc::pack2(__uint_as_float(y[8 * u + 4]), __uint_as_float(y[8 * u + 5]));
      w.w = tc::pack2(__uint_as_float(y[8 * u + 6]), __uint_as_float(y[8 * u + 7]));
      sp[u] = w;
    }
  }
}

// |m| = 0 row block of degree l: partial logits of this warp's 32 channels,
// Lp[q][e][h] += sum_c A[h][l C + c] SiLU(y0_e[l, c]), by warp-level mma.sync on
// 16-edge x 16-channel blocks of SiLU(y0) staged in the warp's tile T (bf16, 16-byte
// pieces of a row swizzled by ((row >> 1) & 3)); each lane owns fixed (e, h) entries.
__device__ __noinline__ void m0_logits(const __nv_bfloat16* Amat, int C, int H, int L, uint32_t tb, int l, int q,
                                       int lane, float* Lp, uint16_t* T, uint32_t T_u32) {
  const int nnt = H > 8 ? 2 : 1;
  uint32_t bf[2][2][2];
#pragma unroll
  for (int kt = 0; kt < 2; ++kt)
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      const int n = nt * 8 + (lane >> 2);
      const int k0 = l * C + q * 32 + kt * 16 + 2 * (lane & 3);
      const bool ok = n < H && nt < nnt;
      const uint32_t* ap = reinterpret_cast<const uint32_t*>(Amat + (size_t)n * L * C + k0);
      bf[kt][nt][0] = ok ? __ldg(ap) : 0u;
      bf[kt][nt][1] = ok ? __ldg(ap + 4) : 0u;
    }
#pragma unroll 1
  for (int j = 0; j < 4; ++j) {
    uint32_t y[32];
    tc::tmem_ld32_issue(tb + 32 * j, y);
    tc::tmem_ld_wait(y);
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const float v = __uint_as_float(y[i]);
      const float sv = __fdividef(v, 1.0f + __expf(-v));
      T[i * 32 + ((((lane >> 3) ^ ((i >> 1) & 3))) << 3) + (lane & 7)] = __bfloat16_as_ushort(__float2bfloat16_rn(sv));
    }
    __syncwarp();
#pragma unroll
    for (int mt = 0; mt < 2; ++mt) {
      uint32_t af[2][4];
#pragma unroll
      for (int kt = 0; kt < 2; ++kt) {
        const int row = 16 * mt + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int chunk = 2 * kt + (lane >> 4);
        tc::ldmatrix_x4(T_u32 + row * 64 + ((chunk ^ ((row >> 1) & 3)) << 4), af[kt]);
      }
#pragma unroll
      for (int nt = 0; nt < 2; ++nt) {
        if (nt < nnt) {
          float lg[4] = {0.f, 0.f, 0.f, 0.f};
          tc::mma_16816(lg, af[0], bf[0][nt]);
          tc::mma_16816(lg, af[1], bf[1][nt]);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int e = 32 * j + 16 * mt + (lane >> 2) + 8 * (r >> 1);
            const int h = 8 * nt + 2 * (lane & 3) + (r & 1);
            if (h < H) Lp[(q * 128 + e) * H + h] += lg[r];
          }
        }
      }
    }
    __syncwarp();
  }
}

// LM = lmax: the degree switches below only instantiate the helpers a launch can reach.
template <int LM>
__global__ void __launch_bounds__(kFThreads, 1) layer_fused_kernel(const __grid_constant__ TcParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = tc::smem_u32(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw_u32);
  const uint32_t X_u32 = base_u32;
  const int nxs = P.f_nxs, nws = P.f_nws;   // x and weight stages of this launch
  const uint32_t W_u32 = base_u32 + nxs * kXBytes;
  EpiSmem* es = reinterpret_cast<EpiSmem*>(base + nxs * kXBytes + nws * kWBytes);
  float* dbuf = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(es) + ((sizeof(EpiSmem) + 15) & ~15));
  int DZ = 0;   // floats of one edge's m = 0 rows of every D^l, each row padded to four floats
  for (int l = 0; l < P.L; ++l) DZ += pad4(2 * l + 1);
  float* m0r = dbuf + 2 * P.f_dgroup;   // [128][DZ]: the tile's m = 0 rows, kept for the whole tile
  FusedCtl* ctl = reinterpret_cast<FusedCtl*>(m0r + 128 * DZ);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &ctl->abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < nxs; ++i) {
      tc::mbar_init(tc::smem_u32(&ctl->x_full[i]), 1);
      tc::mbar_init(tc::smem_u32(&ctl->x_empty[i]), 1);
    }
    for (int i = 0; i < nws; ++i) {
      tc::mbar_init(tc::smem_u32(&ctl->w_full[i]), 1);
      tc::mbar_init(tc::smem_u32(&ctl->w_empty[i]), 1);
    }
    for (int i = 0; i < 2; ++i) {
      tc::mbar_init(tc::smem_u32(&ctl->acc_full[i]), 1);
      tc::mbar_init(tc::smem_u32(&ctl->acc_empty[i]), 256);
    }
    tc::mbar_init(tc::smem_u32(&ctl->mma_done), 1);
    ctl->abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(&ctl->tmem_base), 512);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const long long E = P.n_edges;

  if (warp == 0) {
    // ---------------- bulk copies: weight tiles and the rotate kernel's x tiles ----------------
    if (lane == 0) {
      // x tiles stay in L2 until the last pass of their |m| block reads them; the weight
      // image is read by every CTA and stays too
      const uint64_t keep = tc::policy_evict_last(), drop = tc::policy_evict_first();
      uint32_t ix = 0, iw = 0;
      for (int t = P.t_begin + blockIdx.x; t < P.t_end && !*abort; t += gridDim.x) {
        const uint8_t* xt = P.X + (long long)(t - P.t_begin) * P.nch * 16384;
        for (int p = 0; p < P.npass && !*abort; ++p) {
          const TcPass& ps = P.pass[p];
          const uint32_t bytes = (uint32_t)ps.n * 128u;
          const int nx = ps.block > 0 ? 2 : 1;
          const bool last_of_block = p + 1 == P.npass || P.pass[p + 1].block != ps.block;
          const uint64_t xpol = last_of_block ? drop : keep;
          for (int kb = 0; kb < ps.nk && !*abort; ++kb, ++iw) {
            const int sw = iw % nws;
            if (!tc::mbar_wait(tc::smem_u32(&ctl->w_empty[sw]), ((iw / nws) & 1) ^ 1, P.status, abort, 64)) break;
            tc::mbar_arrive_expect_tx(tc::smem_u32(&ctl->w_full[sw]), bytes);
            tc::bulk_g2s_hint(W_u32 + sw * kWBytes, P.wprep + ps.boff + (long long)kb * bytes, bytes,
                              tc::smem_u32(&ctl->w_full[sw]), keep);
            for (int h = 0; h < nx; ++h, ++ix) {
              const int sx = ix % nxs;
              if (!tc::mbar_wait(tc::smem_u32(&ctl->x_empty[sx]), ((ix / nxs) & 1) ^ 1, P.status, abort, 64)) break;
              const int id = ps.block == 0 ? kb : P.xbase[ps.block] + 2 * kb + h;
              tc::mbar_arrive_expect_tx(tc::smem_u32(&ctl->x_full[sx]), (uint32_t)kXBytes);
              tc::bulk_g2s_hint(X_u32 + sx * kXBytes, xt + (long long)id * kXBytes, (uint32_t)kXBytes,
                                tc::smem_u32(&ctl->x_full[sx]), xpol);
            }
          }
        }
      }
      // the newest phase of every stage must have landed before the CTA exits
      for (uint32_t k = (iw > (uint32_t)nws ? iw - nws : 0); k < iw; ++k) {
        const uint32_t bar = tc::smem_u32(&ctl->w_full[k % nws]);
        const uint64_t t0 = tc::globaltimer();
        while (!tc::mbar_try_wait(bar, (k / nws) & 1) && tc::globaltimer() - t0 < 2000000000ull) {
        }
      }
      for (uint32_t k = (ix > (uint32_t)nxs ? ix - nxs : 0); k < ix; ++k) {
        const uint32_t bar = tc::smem_u32(&ctl->x_full[k % nxs]);
        const uint64_t t0 = tc::globaltimer();
        while (!tc::mbar_try_wait(bar, (k / nxs) & 1) && tc::globaltimer() - t0 < 2000000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer: D[channels][edges] += W X^T ----------------
    if (lane == 0) {
      const uint32_t id = tc::idesc_bf16(128, 128), id_nega = tc::idesc_bf16(128, 128, false, true);
      uint32_t ix = 0, iw = 0, ip = 0;
      for (int t = P.t_begin + blockIdx.x; t < P.t_end && !*abort; t += gridDim.x) {
        for (int p = 0; p < P.npass && !*abort; ++p, ++ip) {
          const TcPass& ps = P.pass[p];
          const int buf = ip & 1;
          const uint32_t acc_t = tmem + buf * 256;
          if (!tc::mbar_wait(tc::smem_u32(&ctl->acc_empty[buf]), ((ip >> 1) & 1) ^ 1, P.status, abort, 32)) break;
          tc::tc_fence_after();
          if (ps.block > 0) {
            // y+ += W1 x+ - W2 x- (columns 0-127); y- += W2 x+ + W1 x- (columns 128-255)
            for (int kb = 0; kb < ps.nk; ++kb, ++iw, ix += 2) {
              const int sw = iw % nws, sp = ix % nxs, sm = (ix + 1) % nxs;
              if (!tc::mbar_wait(tc::smem_u32(&ctl->w_full[sw]), (iw / nws) & 1, P.status, abort)) break;
              if (!tc::mbar_wait(tc::smem_u32(&ctl->x_full[sp]), (ix / nxs) & 1, P.status, abort)) break;
              if (!tc::mbar_wait(tc::smem_u32(&ctl->x_full[sm]), ((ix + 1) / nxs) & 1, P.status, abort)) break;
              tc::tc_fence_after();
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                const uint64_t w1 = tc::sw128_desc(W_u32 + sw * kWBytes + ks * 32);
                const uint64_t w2 = tc::sw128_desc(W_u32 + sw * kWBytes + 16384 + ks * 32);
                const uint64_t xp = tc::sw128_desc(X_u32 + sp * kXBytes + ks * 32);
                const uint64_t xm = tc::sw128_desc(X_u32 + sm * kXBytes + ks * 32);
                const uint32_t a = (kb > 0 || ks > 0) ? 1u : 0u;
                tc::mma_bf16(acc_t, w1, xp, id, a);
                tc::mma_bf16(acc_t, w2, xm, id_nega, 1u);
                tc::mma_bf16(acc_t + 128, w2, xp, id, a);
                tc::mma_bf16(acc_t + 128, w1, xm, id, 1u);
              }
              tc::mma_commit(tc::smem_u32(&ctl->x_empty[sp]));
              tc::mma_commit(tc::smem_u32(&ctl->x_empty[sm]));
              tc::mma_commit(tc::smem_u32(&ctl->w_empty[sw]));
            }
          } else {
            const int nrb = ps.n / 128;   // one or two degrees of y0
            for (int kb = 0; kb < ps.nk; ++kb, ++iw, ++ix) {
              const int sw = iw % nws, sx = ix % nxs;
              if (!tc::mbar_wait(tc::smem_u32(&ctl->w_full[sw]), (iw / nws) & 1, P.status, abort)) break;
              if (!tc::mbar_wait(tc::smem_u32(&ctl->x_full[sx]), (ix / nxs) & 1, P.status, abort)) break;
              tc::tc_fence_after();
#pragma unroll
              for (int ks = 0; ks < 4; ++ks) {
                const uint64_t xd = tc::sw128_desc(X_u32 + sx * kXBytes + ks * 32);
                for (int rb = 0; rb < nrb; ++rb) {
                  const uint64_t wd = tc::sw128_desc(W_u32 + sw * kWBytes + rb * 16384 + ks * 32);
                  tc::mma_bf16(acc_t + rb * 128, wd, xd, id, (kb > 0 || ks > 0) ? 1u : 0u);
                }
              }
              tc::mma_commit(tc::smem_u32(&ctl->x_empty[sx]));
              tc::mma_commit(tc::smem_u32(&ctl->w_empty[sw]));
            }
          }
          tc::mma_commit(tc::smem_u32(&ctl->acc_full[buf]));
        }
      }
      // every issued MMA must finish before TMEM is released
      tc::mma_commit(tc::smem_u32(&ctl->mma_done));
      const uint64_t t0 = tc::globaltimer();
      while (!tc::mbar_try_wait(tc::smem_u32(&ctl->mma_done), 0) && tc::globaltimer() - t0 < 2000000000ull) {
      }
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: two groups of four warps, thread = output channel c ----------------
    // Group 0 (warps 2-5) and group 1 (warps 6-9) each own a fixed set of degrees l
    // (P.own_b): every accumulator of a degree is written by one thread, so the sums
    // are deterministic.  In the |m| = 0 passes group 0 forms the logits and group 1
    // writes the stash.  Every epilogue thread waits for and releases every pass.
    // Waits ignore the abort flag and time out on their own: every epilogue thread then
    // leaves at the same wait, so none is left at a named barrier.
    volatile int no_abort = 0;
    const int g = (warp - 2) >> 2;                         // epilogue group
    const int q = warp & 3, c = q * 32 + lane;            // TMEM lane quadrant, channel
    const int et = threadIdx.x - 64;                       // 0..255
    const int C = P.C, H = P.H, L = P.L, L2 = P.L2, hh = c / (C / H);
    const uint32_t tl = tmem + ((uint32_t)(q * 32) << 16);
    __nv_bfloat16* stash = P.stash + (size_t)blockIdx.x * L * 128 * C;
    float* dg = dbuf + g * P.f_dgroup;                     // this group's Wigner rows
    const EpiArgs EA{P.slots, P.acc_g, P.C, P.L2, P.rec_floats};
    uint32_t ip = 0;
    bool failed = false;
    for (int t = P.t_begin + blockIdx.x; t < P.t_end && !failed; t += gridDim.x) {
      const long long e0 = (long long)t * 128;
      const int nvalid = (int)(E - e0 < 128 ? E - e0 : 128);
      // ---- destination segments of the tile (group 0 threads: one per edge) ----
      if (et < 128) es->dst[et] = et < nvalid ? P.edge_dst[e0 + et] : -1;
      epi_bar();
      {
        const bool start = et < nvalid && (et == 0 || es->dst[et] != es->dst[et - 1]);
        const unsigned bal = __ballot_sync(0xffffffffu, start);
        if (et < 128 && lane == 0) es->wcnt[et >> 5] = __popc(bal);
        epi_bar();
        if (et < 128) {
          int k = 0;
          for (int w = 0; w < (et >> 5); ++w) k += es->wcnt[w];
          k += __popc(bal & ((1u << lane) - 1u));
          if (start) {
            es->seg_d[k] = es->dst[et];
            es->seg_b[k] = et;
          }
          if (et == 127) {
            const int ns = es->wcnt[0] + es->wcnt[1] + es->wcnt[2] + es->wcnt[3];
            es->nseg = ns;
            es->seg_b[ns] = nvalid;
          }
        }
        epi_bar();
        const int ns = es->nseg;
        if (et < ns) {
          const int d = es->seg_d[et];
          const bool before = et == 0 && P.row_ptr[d] < e0;
          const bool after = et == ns - 1 && P.row_ptr[d + 1] > e0 + 128;
          es->seg_slot[et] = before ? 0 : (after ? 1 : -1);
        }
      }
      // ---- |m| = 0 passes: group 0 SiLU(y0) into the logits, group 1 y0 into the stash ----
      float* Lp = dbuf;   // [4][128][H] partial logits of group 0's warps, then their staging tiles
      if (g == 0) {
        for (int i = lane; i < 128 * H; i += 32) Lp[q * 128 * H + i] = 0.f;
        __syncwarp();
      }
      int p = 0;
      uint16_t* T = reinterpret_cast<uint16_t*>(dbuf + 4 * 128 * H) + q * 32 * 32;
      const uint32_t T_u32 = tc::smem_u32(T);
      for (; p < P.npass && P.pass[p].block == 0; ++p, ++ip) {
        const TcPass& ps = P.pass[p];
        const int buf = ip & 1;
        if (!tc::mbar_wait(tc::smem_u32(&ctl->acc_full[buf]), (ip >> 1) & 1, P.status, &no_abort, 64)) {
          failed = true;
          break;
        }
        tc::tc_fence_after();
        for (int rb = 0; rb < ps.n / 128; ++rb) {
          const int l = ps.n_off / 128 + rb;
          const uint32_t tb = tl + buf * 256 + rb * 128;
          if (g == 1) m0_stash(tb, stash + ((size_t)l * C + c) * 128);
          else m0_logits(P.A, C, H, L, tb, l, q, lane, Lp, T, T_u32);
        }
        tc::tc_fence_before();
        tc::mbar_arrive(tc::smem_u32(&ctl->acc_empty[buf]));
      }
      if (failed) break;
      // ---- logits: sum the four partials, add bA; softmax statistics per (segment, head) ----
      epi_bar();
      if (et < 128) {
        for (int h = 0; h < H; ++h) {
          float a = Lp[et * H + h] + Lp[(128 + et) * H + h] + Lp[(256 + et) * H + h] + Lp[(384 + et) * H + h];
          es->pw[et * 16 + h] = a + __bfloat162float(P.bA[h]);
        }
      }
      epi_bar();
      // ---- rows m = 0 of every D^l for the tile (one edge per thread of group 0), fetched
      // asynchronously while the softmax statistics are formed (Lp is no longer needed) ----
      if (et < nvalid && et < 128) {
        const float* wr = P.wig + (size_t)(e0 + et) * P.wfl;
        const uint32_t dz = tc::smem_u32(m0r + et * DZ);
        int off = 0;
        for (int l = 0; l < L; ++l) {
          const int ml = l < P.mmax ? l : P.mmax, dl = 2 * l + 1;
          const float* row = wr + P.woff[l] + ml * dl;   // row m = 0 of D^l
          for (int m = 0; m < dl; ++m) tc::cp_async4(dz + 4 * (off + m), row + m);
          off += pad4(dl);
        }
      }
      // ---- softmax statistics per (segment, head): one warp per pair, lanes over edges ----
      {
        const int ns = es->nseg, ew = et >> 5;
        for (int pr = ew; pr < ns * H; pr += 8) {
          const int k = pr / H, h = pr - k * H;
          const int b = es->seg_b[k], en = es->seg_b[k + 1];
          float mx = -INFINITY;
          for (int e = b + lane; e < en; e += 32) mx = fmaxf(mx, es->pw[e * 16 + h]);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          float sum = 0.f;
          for (int e = b + lane; e < en; e += 32) {
            const float x = __expf(es->pw[e * 16 + h] - mx);
            es->pw[e * 16 + h] = x;
            sum += x;
          }
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
          if (lane == 0) {
            es->segS[k * 16 + h] = sum;
            const int slot = es->seg_slot[k];
            if (slot >= 0) es->segM[slot * 16 + h] = mx;
          }
        }
      }
      if (et < nvalid && et < 128) tc::cp_async_wait_all();
      epi_bar();
      // ---- y0 contributions (first contribution of each record) and (+m, -m) passes ----
      // The group's y0 step of degree l comes right before the degree's first (+m, -m)
      // pass; the others run while the MMA works on passes the group does not own.
      auto y0_step = [&](int l) {
        int offz = 0;
        for (int q2 = 0; q2 < l; ++q2) offz += pad4(2 * q2 + 1);
        const uint4* st_row = reinterpret_cast<const uint4*>(stash + ((size_t)l * C + c) * 128);
        switch (l) {
          case 0: y0_degree<(LM >= 0 ? 1 : 2 * LM + 1)>(EA, es, m0r, t, l, c, hh, nvalid, DZ, offz, st_row); break;
          case 1: y0_degree<(LM >= 1 ? 3 : 2 * LM + 1)>(EA, es, m0r, t, l, c, hh, nvalid, DZ, offz, st_row); break;
          case 2: y0_degree<(LM >= 2 ? 5 : 2 * LM + 1)>(EA, es, m0r, t, l, c, hh, nvalid, DZ, offz, st_row); break;
          case 3: y0_degree<(LM >= 3 ? 7 : 2 * LM + 1)>(EA, es, m0r, t, l, c, hh, nvalid, DZ, offz, st_row); break;
          case 4: y0_degree<(LM >= 4 ? 9 : 2 * LM + 1)>(EA, es, m0r, t, l, c, hh, nvalid, DZ, offz, st_row); break;
          case 5: y0_degree<(LM >= 5 ? 11 : 2 * LM + 1)>(EA, es, m0r, t, l, c, hh, nvalid, DZ, offz, st_row); break;
          default: y0_degree<(LM >= 6 ? 13 : 2 * LM + 1)>(EA, es, m0r, t, l, c, hh, nvalid, DZ, offz, st_row); break;
        }
      };
      unsigned y0_left = 0;
      for (int l = 0; l < L; ++l)
        if (own_deg(P, g, l)) y0_left |= 1u << l;
      // ---- (+m, -m) passes: each processed by the group owning its degree ----
      // The group's Wigner rows (l, +b), (l, -b) of a pass sit in dg as [e][2][pad4(2l+1)]
      // (one or two buffers); the next own pass's rows are fetched asynchronously while
      // the current pass is summed when both fit.
      const int pass_floats = 128 * 2 * pad4(2 * L - 1);
      const bool dbl = 2 * pass_floats <= P.f_dgroup;
      int pown = p;
      while (pown < P.npass && !own_deg(P, g, pass_l(P, pown))) ++pown;
      int half = 0;
      if (pown < P.npass) {
        fetch_rows(P, pown, dg, et & 127, nvalid, e0);
        tc::cp_async_wait_all();
      }
      group_bar(g);
      for (; p < P.npass; ++p, ++ip) {
        const int buf = ip & 1;
        const int l = pass_l(P, p);
        if (own_deg(P, g, l)) {
          if ((y0_left >> l) & 1u) {
            y0_step(l);
            y0_left &= ~(1u << l);
          }
        } else if (y0_left) {
          // the degree of the group's next own pass if still pending, else the lowest
          const int po = next_own(P, g, p);
          int ly = po < P.npass ? pass_l(P, po) : -1;
          if (ly < 0 || !((y0_left >> ly) & 1u)) ly = __ffs(y0_left) - 1;
          y0_step(ly);
          y0_left &= ~(1u << ly);
        }
        if (!tc::mbar_wait(tc::smem_u32(&ctl->acc_full[buf]), (ip >> 1) & 1, P.status, &no_abort, 64)) {
          failed = true;
          break;
        }
        if (own_deg(P, g, l)) {
          const int pn = next_own(P, g, p);
          float* dcur = dg + half * (dbl ? pass_floats : 0);
          if (dbl && pn < P.npass) fetch_rows(P, pn, dg + (half ^ 1) * pass_floats, et & 127, nvalid, e0);
          tc::tc_fence_after();
          const uint32_t tb = tl + buf * 256;
          switch (l) {
            case 1: pm_degree<(LM >= 1 ? 3 : 2 * LM + 1)>(EA, es, dcur, t, l, c, hh, nvalid, tb); break;
            case 2: pm_degree<(LM >= 2 ? 5 : 2 * LM + 1)>(EA, es, dcur, t, l, c, hh, nvalid, tb); break;
            case 3: pm_degree<(LM >= 3 ? 7 : 2 * LM + 1)>(EA, es, dcur, t, l, c, hh, nvalid, tb); break;
            case 4: pm_degree<(LM >= 4 ? 9 : 2 * LM + 1)>(EA, es, dcur, t, l, c, hh, nvalid, tb); break;
            case 5: pm_degree<(LM >= 5 ? 11 : 2 * LM + 1)>(EA, es, dcur, t, l, c, hh, nvalid, tb); break;
            default: pm_degree<(LM >= 6 ? 13 : 2 * LM + 1)>(EA, es, dcur, t, l, c, hh, nvalid, tb); break;
          }
          tc::tc_fence_before();
          tc::mbar_arrive(tc::smem_u32(&ctl->acc_empty[buf]));
          if (pn < P.npass) {
            if (!dbl) {
              group_bar(g);   // every thread of the group is done with the rows
              fetch_rows(P, pn, dg, et & 127, nvalid, e0);
            }
            tc::cp_async_wait_all();
            group_bar(g);
            half ^= dbl ? 1 : 0;
          }
        } else {
          tc::mbar_arrive(tc::smem_u32(&ctl->acc_empty[buf]));
        }
      }
      if (failed) break;
      while (y0_left) {   // degrees without (+m, -m) passes, or not yet reached
        const int ly = __ffs(y0_left) - 1;
        y0_step(ly);
        y0_left &= ~(1u << ly);
      }
      asm volatile("" ::: "memory");   // the record reads below follow this thread's adds
      // ---- finish the destinations whose edges all lie in this tile (rows of own degrees) ----
      {
        const int ns = es->nseg;
        for (int k = 0; k < ns; ++k) {
          const int slot = es->seg_slot[k];
          if (slot < 0) {
            const int d = es->seg_d[k];
            const float inv = 1.0f / es->segS[k * 16 + hh];
            const size_t o = (size_t)d * L2 * C + c;
            const float* ag = P.acc_g + o;
            for (int l = 0; l < L; ++l) {
              if (!own_deg(P, g, l)) continue;
              for (int i = l * l; i < (l + 1) * (l + 1); ++i) {
                const float v = __bfloat162float(P.node_in[o + (size_t)i * C]) + ag[(size_t)i * C] * inv;
                P.node_out[o + (size_t)i * C] = __float2bfloat16_rn(v);
              }
            }
          } else if (et < H) {
            float* rec = P.slots + ((size_t)t * 2 + slot) * P.rec_floats + (size_t)L2 * C;
            rec[et] = es->segM[slot * 16 + et];
            rec[16 + et] = es->segS[k * 16 + et];
          }
        }
      }
      epi_bar();   // the next tile rewrites the segment table, logits and weights
    }
    if (failed) {
      egnn_flag(P.status, EGNN_DEV_WAIT_TIMEOUT);
      *abort = 1;
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, 512);
  }
}

// Destinations the fused kernel did not finish: atoms without incoming edges keep
// their embedding; atoms whose edges cross tile boundaries merge their per-tile
// records (softmax maxima and sums rescaled to the common maximum).  One CTA of C
// threads (thread = channel) per atom.
__global__ void __launch_bounds__(128, 8) combine_kernel(const __grid_constant__ TcParams P) {
  const int d = blockIdx.x, c = threadIdx.x;
  const int C = P.C, L2 = P.L2, hh = c / (C / P.H);
  const size_t o = (size_t)d * L2 * C + c;
  const int b = P.row_ptr[d], en = P.row_ptr[d + 1];
  if (en <= b) {
    for (int i = 0; i < L2; ++i) P.node_out[o + (size_t)i * C] = P.node_in[o + (size_t)i * C];
    return;
  }
  const int t0 = b >> 7, t1 = (en - 1) >> 7;
  if (t0 == t1) return;
  const size_t rf = P.rec_floats;
  auto record = [&](int t) { return P.slots + ((size_t)t * 2 + (t == t0 ? 1 : 0)) * rf; };
  float mx = -INFINITY;
  for (int t = t0; t <= t1; ++t) mx = fmaxf(mx, record(t)[(size_t)L2 * C + hh]);
  float sum = 0.f;
  for (int t = t0; t <= t1; ++t) {
    const float* rec = record(t) + (size_t)L2 * C;
    sum += __expf(rec[hh] - mx) * rec[16 + hh];
  }
  const float inv = 1.0f / sum;
  // rows in chunks of 8: few registers, so many atoms are in flight per SM
  for (int i0 = 0; i0 < L2; i0 += 8) {
    float acc[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) acc[i] = 0.f;
    for (int t = t0; t <= t1; ++t) {
      const float* rec = record(t);
      const float w = __expf(rec[(size_t)L2 * C + hh] - mx);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        if (i0 + i < L2) acc[i] += w * rec[(size_t)(i0 + i) * C + c];
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (i0 + i < L2)
        P.node_out[o + (size_t)(i0 + i) * C] =
            __float2bfloat16_rn(__bfloat162float(P.node_in[o + (size_t)(i0 + i) * C]) + acc[i] * inv);
  }
}

// Destination atom of every edge (one warp per atom; consecutive edges, coalesced stores).
__global__ void edge_dst_kernel(const int32_t* __restrict__ row_ptr, int n_atoms, int32_t* __restrict__ dst) {
  const int d = (blockIdx.x * blockDim.x + threadIdx.x) >> 5, lane = threadIdx.x & 31;
  if (d >= n_atoms) return;
  for (int e = row_ptr[d] + lane; e < row_ptr[d + 1]; e += 32) dst[e] = d;
}

// Shared memory of one launch: x stages, weight stages, EpiSmem, dbuf, control block
// (+ 1 KB to align the operand stages to 1024 bytes).
size_t fused_smem_bytes(int nxs, int nws, int dgroup, int L) {
  int DZ = 0;
  for (int l = 0; l < L; ++l) DZ += ((2 * l + 1) + 3) & ~3;
  return (size_t)nxs * kXBytes + (size_t)nws * kWBytes + ((sizeof(EpiSmem) + 15) & ~(size_t)15) +
         sizeof(float) * (2 * (size_t)dgroup + 128 * (size_t)DZ) + sizeof(FusedCtl) + 1024;
}

#ifndef EGNN_FUSED_DOUBLE_ROWS
#define EGNN_FUSED_DOUBLE_ROWS 0
#endif

// dbuf size and x stage count: dbuf holds the largest of its three uses (partial logits
// and staging tiles, the m = 0 rows of a tile, each group's pass rows, single- or
// double-buffered); the x stages take what shared memory is left, up to kMaxXS.
bool fused_layout(const TcParams& P, int& nxs, int& nws, int& dgroup) {
  int DZ = 0;   // floats of one edge's m = 0 rows, each row padded to four floats
  for (int l = 0; l < P.L; ++l) DZ += ((2 * l + 1) + 3) & ~3;
  (void)DZ;   // the m = 0 rows have their own region after dbuf
  const int need_lp = 4 * 128 * P.H + 4 * 32 * 32 / 2;       // partial logits + bf16 tiles
  const int pass_floats = 128 * 2 * (((2 * P.L - 1) + 3) & ~3);
  const int need_rows = (EGNN_FUSED_DOUBLE_ROWS ? 4 : 2) * pass_floats;
  int dbuf = need_lp > need_rows ? need_lp : need_rows;
  dbuf = (dbuf + 7) & ~7;
  dgroup = dbuf / 2;
  int dev = 0, optin = 232448;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  // three weight stages with at least four x stages, else two weight stages
  for (nws = kMaxWS; nws >= 2; --nws)
    for (nxs = kMaxXS; nxs >= (nws == kMaxWS ? 4 : 3); --nxs)
      if (fused_smem_bytes(nxs, nws, dgroup, P.L) <= (size_t)optin) return true;
  return false;
}

cudaError_t fused_consumer(const TcParams& Ps, int grid, cudaStream_t st, void*) {
  const size_t sm = fused_smem_bytes(Ps.f_nxs, Ps.f_nws, Ps.f_dgroup, Ps.L);
  cudaError_t err = cudaSuccess;
  switch (Ps.lmax) {
#define EGNN_FUSED_CASE(LMv)                                                                             \
  case LMv:                                                                                              \
    err = cudaFuncSetAttribute(layer_fused_kernel<LMv>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm); \
    if (err != cudaSuccess) return err;                                                                  \
    layer_fused_kernel<LMv><<<grid, kFThreads, sm, st>>>(Ps);                                           \
    break;
    EGNN_FUSED_CASE(1) EGNN_FUSED_CASE(2) EGNN_FUSED_CASE(3) EGNN_FUSED_CASE(4) EGNN_FUSED_CASE(5) EGNN_FUSED_CASE(6)
#undef EGNN_FUSED_CASE
    default:
      return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

// Destination of every edge, weight prep, then per range of edge tiles: gates and rotation
// -> fused SO(2) layer; then the destinations that cross tile boundaries or have none.
cudaError_t launch_layer_fused(const TcParams& P0, const TcWeights& W, cudaStream_t st) {
  TcParams P = P0;
  if (!fused_layout(P, P.f_nxs, P.f_nws, P.f_dgroup)) return cudaErrorInvalidValue;
  if (P.n_edges > 0) edge_dst_kernel<<<(P.n_atoms * 32 + 255) / 256, 256, 0, st>>>(P.row_ptr, P.n_atoms, P.edge_dst);
  cudaError_t err = launch_tc_pipeline(P, W, st, fused_consumer, nullptr, true);
  if (err != cudaSuccess) return err;
  combine_kernel<<<P.n_atoms, 128, 0, st>>>(P);
  return cudaGetLastError();
}
