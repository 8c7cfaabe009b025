// Tensor-core (tcgen05) eSCN layer for bf16 embeddings, C = 128, mmax <= 2, lmax <= 6.
//
// Method: "MALOQ: Massively Accelerated Learning of Operators for Quantum
// Transport", Sections II-B1 and III (rotate each edge onto one axis so the
// SO(3) interaction becomes SO(2) "constrained linear layers", then aggregate
// onto the target atom), Section III-D / Fig. 4(b) (message from the
// concatenated pair n_s (+) n_d); incoming-edge ownership from the review page
// of "Distributed Equivariant Graph Neural Networks for Large-Scale Electronic
// Structure Prediction", "What carries the argument".  MALOQ builds its
// Wigner-D matrices with Triton block-packed tl.dot on Hopper (Fig. 3(d));
// here the contractions that are GEMMs run on tcgen05 and the small per-edge
// rotations stay on the CUDA cores that feed them.
//
// Three launches per layer:
//   prep_weights  packs the gate and SO(2) weight matrices into the exact
//                 shared-memory image of K-major 128-byte-swizzled B tiles, one
//                 tile per (pass, 64-wide K chunk), so one 1-D bulk copy moves it.
//   so2_tc        persistent; per tile of 128 consecutive edges (one edge per
//                 TMEM lane) it runs a list of passes, each a GEMM
//                 D[128 x N<=512] = A[128 x K] B[N x K]^T accumulated in TMEM:
//                   gate passes  A = SiLU(W1 rho(|r_e|) + b1), B = W2 -> gate g_e
//                                (+ b2, bf16) into a per-CTA scratch;
//                   SO(2) passes A = g_e * (D^l(R_e) [n_s || n_d]) rows |m| = b
//                                built on the fly, B = W0 (b = 0) or the real
//                                form [[W_b1, -W_b2], [W_b2, W_b1]] (b > 0)
//                                -> y_e (bf16) and the attention logits from
//                                SiLU(y0).
//                 Warp roles: 0 bulk-copies B tiles, 1 issues MMAs (one thread)
//                 and owns TMEM, 2-5 build A tiles, 6-9 drain TMEM.
//   agg           one CTA per destination atom, thread = channel: softmax of the
//                 logits over the atom's incoming edges, rotate y back with the
//                 kept rows of D^l(R_e), weighted sum, residual; no atomics.
#include <math.h>

#include "common.cuh"
#include "so2_params.cuh"
#include "so2_tc.cuh"
#include "tc_ptx.cuh"

namespace {

constexpr int kSA = 4;                 // A stages (128 x 64 bf16 = 16 KB each)
constexpr int kSB = 2;                 // B stages (<= 512 x 64 bf16 = 64 KB each)
constexpr int kAStage = 128 * 128;
constexpr int kBStage = 512 * 128;
constexpr int kThreads = 448;   // 0 loader, 1 MMA, 2-9 producers, 10-13 epilogue
constexpr int kProducers = 256;
constexpr int kTmemCols = 512;

struct SmemCtl {
  uint64_t a_full[kSA], a_empty[kSA], b_full[kSB], b_empty[kSB];
  uint64_t acc_full, acc_empty, gate_ready, mma_done;
  uint32_t tmem_base;
  int abort;
};

__device__ __forceinline__ void unpack8(const uint4& q, float* f) {
  const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xffff0000u);
  }
}

__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// acc[i] (+)= sum_{mp < dl} co[mp] * z[mp*C + i], i < 32; loads are issued three
// rows (12 x 16 B) at a time before their FMAs so that more of them are in flight.
__device__ __forceinline__ void rot_acc1(float* acc, const __nv_bfloat16* z, int C, const float* co, int dl) {
  for (int mp0 = 0; mp0 < dl; mp0 += 3) {
    uint4 q[3][4];
    float c[3];
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      const bool ok = mp0 + u < dl;
      const uint4* zp = reinterpret_cast<const uint4*>(z + (ok ? mp0 + u : 0) * C);
#pragma unroll
      for (int k = 0; k < 4; ++k) q[u][k] = ok ? __ldg(zp + k) : make_uint4(0, 0, 0, 0);
      c[u] = ok ? __ldg(co + mp0 + u) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 3; ++u)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float f[8];
        unpack8(q[u][k], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[8 * k + i] += c[u] * f[i];
      }
  }
}

// Same for two coefficient rows at once (the +b and -b rows share z), two rows of z
// (8 x 16 B) in flight per batch.
__device__ __forceinline__ void rot_acc2(float* ap, float* am, const __nv_bfloat16* z, int C, const float* cop,
                                         const float* com, int dl) {
  for (int mp0 = 0; mp0 < dl; mp0 += 2) {
    uint4 q[2][4];
    float cp[2], cm[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const bool ok = mp0 + u < dl;
      const uint4* zp = reinterpret_cast<const uint4*>(z + (ok ? mp0 + u : 0) * C);
#pragma unroll
      for (int k = 0; k < 4; ++k) q[u][k] = ok ? __ldg(zp + k) : make_uint4(0, 0, 0, 0);
      cp[u] = ok ? __ldg(cop + mp0 + u) : 0.f;
      cm[u] = ok ? __ldg(com + mp0 + u) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        float f[8];
        unpack8(q[u][k], f);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          ap[8 * k + i] += cp[u] * f[i];
          am[8 * k + i] += cm[u] * f[i];
        }
      }
  }
}

// Writes 32 values (columns [32*half, 32*half+32) of a 64-wide K chunk) of row r
// into a 128B-swizzled K-major tile.
__device__ __forceinline__ void store_row32(uint8_t* tile, int r, int half, const float* v) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    int chunk = half * 4 + q;
    uint4 w;
    w.x = pack2(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack2(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack2(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack2(v[8 * q + 6], v[8 * q + 7]);
    *reinterpret_cast<uint4*>(tile + r * 128 + ((chunk ^ (r & 7)) << 4)) = w;
  }
}

__global__ void __launch_bounds__(kThreads, 1) so2_tc_kernel(const __grid_constant__ TcParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = tc::smem_u32(smem_raw);
  const uint32_t base_u32 = (raw_u32 + 1023u) & ~1023u;
  uint8_t* base = smem_raw + (base_u32 - raw_u32);
  uint8_t* Abuf = base;
  uint8_t* Bbuf = base + kSA * kAStage;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(Bbuf + kSB * kBStage);
  const uint32_t A_u32 = base_u32;
  const uint32_t B_u32 = base_u32 + kSA * kAStage;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  volatile int* abort = &ctl->abort;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kSA; ++i) {
      tc::mbar_init(tc::smem_u32(&ctl->a_full[i]), kProducers);
      tc::mbar_init(tc::smem_u32(&ctl->a_empty[i]), 1);
    }
    for (int i = 0; i < kSB; ++i) {
      tc::mbar_init(tc::smem_u32(&ctl->b_full[i]), 1);
      tc::mbar_init(tc::smem_u32(&ctl->b_empty[i]), 1);
    }
    tc::mbar_init(tc::smem_u32(&ctl->acc_full), 1);
    tc::mbar_init(tc::smem_u32(&ctl->acc_empty), 128);
    tc::mbar_init(tc::smem_u32(&ctl->gate_ready), 128);
    tc::mbar_init(tc::smem_u32(&ctl->mma_done), 1);
    ctl->abort = 0;
    tc::fence_barrier_init();
  }
  if (warp == 1) {
    tc::tmem_alloc(tc::smem_u32(&ctl->tmem_base), kTmemCols);
    tc::tmem_relinquish();
  }
  tc::tc_fence_before();
  __syncthreads();
  tc::tc_fence_after();
  const uint32_t tmem = ctl->tmem_base;
  const int L = P.L, C = P.C, H = P.H, K = P.K;
  const int C2 = 2 * C;
  const long long E = P.n_edges;

  if (warp == 0) {
    // ---------------- B loader ----------------
    if (lane == 0) {
      uint32_t ib = 0;
      for (int t = blockIdx.x; t < P.n_tiles && !*abort; t += gridDim.x) {
        for (int p = 0; p < P.npass && !*abort; ++p) {
          const TcPass& ps = P.pass[p];
          const uint32_t bytes = (uint32_t)ps.n * 128u;
          for (int j = 0; j < ps.nk; ++j, ++ib) {
            int sb = ib % kSB;
            if (!tc::mbar_wait(tc::smem_u32(&ctl->b_empty[sb]), ((ib / kSB) & 1) ^ 1, P.status, abort)) break;
            tc::mbar_arrive_expect_tx(tc::smem_u32(&ctl->b_full[sb]), bytes);
            tc::bulk_g2s(B_u32 + sb * kBStage, P.wprep + ps.boff + (long long)j * bytes, bytes,
                         tc::smem_u32(&ctl->b_full[sb]));
          }
        }
      }
      // drain: the newest phase of each stage must have landed before the CTA exits
      for (uint32_t k = (ib > (uint32_t)kSB ? ib - kSB : 0); k < ib; ++k) {
        uint32_t bar = tc::smem_u32(&ctl->b_full[k % kSB]);
        uint64_t t0 = tc::globaltimer();
        while (!tc::mbar_try_wait(bar, (k / kSB) & 1) && tc::globaltimer() - t0 < 2000000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      uint32_t ia = 0, ib = 0, ip = 0;
      for (int t = blockIdx.x; t < P.n_tiles && !*abort; t += gridDim.x) {
        for (int p = 0; p < P.npass && !*abort; ++p, ++ip) {
          const TcPass& ps = P.pass[p];
          if (!tc::mbar_wait(tc::smem_u32(&ctl->acc_empty), (ip & 1) ^ 1, P.status, abort)) break;
          tc::tc_fence_after();
          for (int j = 0; j < ps.nk; ++j, ++ia, ++ib) {
            int sa = ia % kSA, sb = ib % kSB;
            if (!tc::mbar_wait(tc::smem_u32(&ctl->a_full[sa]), (ia / kSA) & 1, P.status, abort)) break;
            if (!tc::mbar_wait(tc::smem_u32(&ctl->b_full[sb]), (ib / kSB) & 1, P.status, abort)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              uint64_t ad = tc::sw128_desc(A_u32 + sa * kAStage + ks * 32);
              for (int n0 = 0; n0 < ps.n; n0 += 256) {
                int ns = ps.n - n0 < 256 ? ps.n - n0 : 256;
                uint64_t bd = tc::sw128_desc(B_u32 + sb * kBStage + n0 * 128 + ks * 32);
                tc::mma_bf16(tmem + n0, ad, bd, tc::idesc_bf16(128, ns), (j > 0 || ks > 0) ? 1u : 0u);
              }
            }
            tc::mma_commit(tc::smem_u32(&ctl->a_empty[sa]));
            tc::mma_commit(tc::smem_u32(&ctl->b_empty[sb]));
          }
          tc::mma_commit(tc::smem_u32(&ctl->acc_full));
        }
      }
      // every issued MMA must finish before TMEM is released
      tc::mma_commit(tc::smem_u32(&ctl->mma_done));
      uint64_t t0 = tc::globaltimer();
      while (!tc::mbar_try_wait(tc::smem_u32(&ctl->mma_done), 0) && tc::globaltimer() - t0 < 2000000000ull) {
      }
    }
    __syncwarp();
  } else if (warp >= 2 && warp < 10) {
    // ---------------- A producers: thread = (tile row = edge, 32-channel half) ----------------
    const int pidx = (warp - 2) * 32 + lane;
    const int r = pidx & 127;
    const int half = pidx >> 7;
    const __nv_bfloat16* gsc = P.gate_scratch + ((long long)blockIdx.x * 128 + r) * P.gcols;
    uint32_t ia = 0, it = 0;
    for (int t = blockIdx.x; t < P.n_tiles && !*abort; t += gridDim.x, ++it) {
      const long long e = (long long)t * 128 + r;
      const bool valid = e < E;
      int s = 0, d = 0;
      float dist = 0.f;
      if (valid) {
        s = P.src[e];
        int lo = 0, hi = P.n_atoms;
        while (hi - lo > 1) {
          int mid = (lo + hi) >> 1;
          if (P.row_ptr[mid] <= e) lo = mid; else hi = mid;
        }
        d = lo;
        if (s < 0 || s >= P.n_atoms) {
          egnn_flag(P.status, EGNN_DEV_INDEX_RANGE);
          s = d;
        }
        dist = P.dist[e];
      }
      const float* De = P.wig + (valid ? e : 0) * (long long)P.wfl;
      bool gate_waited = false;
      for (int p = 0; p < P.npass && !*abort; ++p) {
        const TcPass& ps = P.pass[p];
        if (ps.kind == 0) {
          // hidden layer of the radial MLP, 64 channels per chunk
          const float mu_step = P.rcut / (float)(K - 1);
          const float inv2s2 = 1.0f / (2.0f * mu_step * mu_step);
          for (int j = 0; j < ps.nk; ++j, ++ia) {
            int sa = ia % kSA;
            if (!tc::mbar_wait(tc::smem_u32(&ctl->a_empty[sa]), ((ia / kSA) & 1) ^ 1, P.status, abort)) break;
            uint8_t* tile = Abuf + sa * kAStage;
            {
              float v[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) v[i] = 0.f;
              if (valid) {
                const int c0 = j * 64 + half * 32;
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = __bfloat162float(P.b1[c0 + i]);
                for (int k = 0; k < K; ++k) {
                  float dd = dist - k * mu_step;
                  float rho = __expf(-dd * dd * inv2s2);
#pragma unroll
                  for (int i = 0; i < 32; ++i) v[i] += __bfloat162float(P.W1[(c0 + i) * K + k]) * rho;
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = v[i] / (1.0f + __expf(-v[i]));
              }
              store_row32(tile, r, half, v);
            }
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(tc::smem_u32(&ctl->a_full[sa]));
          }
          continue;
        }
        if (!gate_waited) {
          if (!tc::mbar_wait(tc::smem_u32(&ctl->gate_ready), it & 1, P.status, abort)) break;
          gate_waited = true;
        }
        const int b = ps.block;
        if (b == 0) {
          for (int j = 0; j < ps.nk; ++j, ++ia) {
            int sa = ia % kSA;
            if (!tc::mbar_wait(tc::smem_u32(&ctl->a_empty[sa]), ((ia / kSA) & 1) ^ 1, P.status, abort)) break;
            uint8_t* tile = Abuf + sa * kAStage;
            const int l = j / (C2 / 64), c2b = j % (C2 / 64);
            const int dl = 2 * l + 1, ml = l < P.mmax ? l : P.mmax;
            const float* Drow = De + P.woff[l] + ml * dl;          // row m = 0
            const int cs = c2b * 64;
            const __nv_bfloat16* z = (cs < C) ? P.node_in + ((long long)s * P.L2 + l * l) * C + cs
                                              : P.node_in + ((long long)d * P.L2 + l * l) * C + (cs - C);
            {
              float acc[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) acc[i] = 0.f;
              if (valid) {
                rot_acc1(acc, z + half * 32, C, Drow, dl);
                const uint4* gp = reinterpret_cast<const uint4*>(gsc + l * C2 + cs + half * 32);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  float f[8];
                  unpack8(gp[q], f);
#pragma unroll
                  for (int i = 0; i < 8; ++i) acc[8 * q + i] *= f[i];
                }
              }
              store_row32(tile, r, half, acc);
            }
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(tc::smem_u32(&ctl->a_full[sa]));
          }
        } else {
          // chunk pairs (+b, -b) of the same (l, 64 channels): z is read once for both
          for (int j = 0; j < ps.nk; j += 2, ia += 2) {
            int sa0 = ia % kSA, sa1 = (ia + 1) % kSA;
            if (!tc::mbar_wait(tc::smem_u32(&ctl->a_empty[sa0]), ((ia / kSA) & 1) ^ 1, P.status, abort)) break;
            if (!tc::mbar_wait(tc::smem_u32(&ctl->a_empty[sa1]), (((ia + 1) / kSA) & 1) ^ 1, P.status, abort))
              break;
            uint8_t* tp = Abuf + sa0 * kAStage;
            uint8_t* tm = Abuf + sa1 * kAStage;
            const int q2 = j >> 1;
            const int l = b + q2 / (C2 / 64), c2b = q2 % (C2 / 64);
            const int dl = 2 * l + 1, ml = l < P.mmax ? l : P.mmax;
            const float* Dp = De + P.woff[l] + (ml + b) * dl;
            const float* Dm = De + P.woff[l] + (ml - b) * dl;
            const int cs = c2b * 64;
            const __nv_bfloat16* z = (cs < C) ? P.node_in + ((long long)s * P.L2 + l * l) * C + cs
                                              : P.node_in + ((long long)d * P.L2 + l * l) * C + (cs - C);
            {
              float ap[32], am[32];
#pragma unroll
              for (int i = 0; i < 32; ++i) ap[i] = am[i] = 0.f;
              if (valid) {
                rot_acc2(ap, am, z + half * 32, C, Dp, Dm, dl);
                const uint4* gp = reinterpret_cast<const uint4*>(gsc + l * C2 + cs + half * 32);
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                  float f[8];
                  unpack8(gp[q], f);
#pragma unroll
                  for (int i = 0; i < 8; ++i) {
                    ap[8 * q + i] *= f[i];
                    am[8 * q + i] *= f[i];
                  }
                }
              }
              store_row32(tp, r, half, ap);
              store_row32(tm, r, half, am);
            }
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(tc::smem_u32(&ctl->a_full[sa0]));
            tc::mbar_arrive(tc::smem_u32(&ctl->a_full[sa1]));
          }
        }
      }
    }
  } else {
    // ---------------- epilogue: thread = TMEM lane = edge ----------------
    const int sub = warp & 3;
    const int r = sub * 32 + lane;
    const uint32_t tl = tmem + ((uint32_t)(sub * 32) << 16);
    __nv_bfloat16* gsc = P.gate_scratch + ((long long)blockIdx.x * 128 + r) * P.gcols;
    uint32_t ip = 0;
    for (int t = blockIdx.x; t < P.n_tiles && !*abort; t += gridDim.x) {
      const long long e = (long long)t * 128 + r;
      const bool valid = e < E;
      float lg[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) lg[h] = 0.f;
      for (int p = 0; p < P.npass && !*abort; ++p, ++ip) {
        const TcPass& ps = P.pass[p];
        if (!tc::mbar_wait(tc::smem_u32(&ctl->acc_full), ip & 1, P.status, abort)) break;
        tc::tc_fence_after();
        for (int g = 0; g < ps.n; g += 32) {
          float v[32];
          tc::tmem_ld32(tl + g, v);
          const int col = ps.n_off + g;
          if (ps.kind == 0) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] += __bfloat162float(P.b2[col + i]);
            uint4* dst = reinterpret_cast<uint4*>(gsc + col);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(pack2(v[8 * q], v[8 * q + 1]), pack2(v[8 * q + 2], v[8 * q + 3]),
                                  pack2(v[8 * q + 4], v[8 * q + 5]), pack2(v[8 * q + 6], v[8 * q + 7]));
          } else if (valid) {
            uint4* dst = reinterpret_cast<uint4*>(P.Y + e * (long long)P.ncols_y + P.ybase[ps.block] + col);
#pragma unroll
            for (int q = 0; q < 4; ++q)
              dst[q] = make_uint4(pack2(v[8 * q], v[8 * q + 1]), pack2(v[8 * q + 2], v[8 * q + 3]),
                                  pack2(v[8 * q + 4], v[8 * q + 5]), pack2(v[8 * q + 6], v[8 * q + 7]));
            if (ps.block == 0 && P.with_logits) {
              for (int h = 0; h < H; ++h) {
                const __nv_bfloat16* Ah = P.A + (long long)h * L * C + col;
                float a = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) a += __bfloat162float(Ah[i]) * (v[i] / (1.0f + __expf(-v[i])));
                lg[h] += a;
              }
            }
          }
        }
        tc::tc_fence_before();
        tc::mbar_arrive(tc::smem_u32(&ctl->acc_empty));
        if (ps.kind == 0 && ps.last_of_kind) tc::mbar_arrive(tc::smem_u32(&ctl->gate_ready));
        if (ps.kind == 1 && ps.block == 0 && ps.last_of_kind && valid && P.with_logits) {
          for (int h = 0; h < H; ++h) P.logits[e * H + h] = lg[h] + __bfloat162float(P.bA[h]);
        }
      }
    }
  }
  tc::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc::tc_fence_after();
    tc::tmem_dealloc(tmem, kTmemCols);
  }
}

// One thread per element of the prepared weight image.
__global__ void prep_weights_kernel(const __grid_constant__ TcParams P, const __nv_bfloat16* __restrict__ W2,
                                    const __nv_bfloat16* __restrict__ W0,
                                    const __nv_bfloat16* __restrict__ Wm1a, const __nv_bfloat16* __restrict__ Wm1b,
                                    const __nv_bfloat16* __restrict__ Wm2a, const __nv_bfloat16* __restrict__ Wm2b,
                                    long long total_elems, uint8_t* __restrict__ out) {
  long long idx = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= total_elems) return;
  const int C = P.C, C2 = 2 * P.C, L = P.L;
  // locate the pass
  long long off = idx * 2;   // byte offset
  int p = 0;
  while (p + 1 < P.npass && P.pass[p + 1].boff <= off) ++p;
  const TcPass& ps = P.pass[p];
  long long rel = off - ps.boff;
  const long long tile_bytes = (long long)ps.n * 128;
  int j = (int)(rel / tile_bytes);
  int rem = (int)(rel - (long long)j * tile_bytes);
  int r = rem / 128;
  int pos = rem % 128;
  int chunk_pos = pos >> 4;
  int chunk = chunk_pos ^ (r & 7);
  int k = chunk * 8 + ((pos & 15) >> 1);
  int row = ps.n_off + r;   // output row of the block matrix
  float v = 0.f;
  if (ps.kind == 0) {
    v = __bfloat162float(W2[(long long)row * C + j * 64 + k]);
  } else if (ps.block == 0) {
    v = __bfloat162float(W0[(long long)row * (L * C2) + j * 64 + k]);
  } else {
    const int b = ps.block, nb = L - b;
    const __nv_bfloat16* Wa = b == 1 ? Wm1a : Wm2a;
    const __nv_bfloat16* Wb = b == 1 ? Wm1b : Wm2b;
    const int q2 = j >> 1, sgn = j & 1;
    const int lq = q2 / (C2 / 64), c2b = q2 % (C2 / 64);
    const int kg = lq * C2 + c2b * 64 + k;        // index inside x+ or x-
    const int ld = nb * C2;
    if (row < nb * C) {                                // y+ = W_b1 x+ - W_b2 x-
      v = sgn == 0 ? __bfloat162float(Wa[(long long)row * ld + kg]) : -__bfloat162float(Wb[(long long)row * ld + kg]);
    } else {                                           // y- = W_b2 x+ + W_b1 x-
      int o = row - nb * C;
      v = sgn == 0 ? __bfloat162float(Wb[(long long)o * ld + kg]) : __bfloat162float(Wa[(long long)o * ld + kg]);
    }
  }
  reinterpret_cast<__nv_bfloat16*>(out)[idx] = __float2bfloat16_rn(v);
}

// Aggregation: one CTA per destination atom, thread = channel.  Softmax statistics
// per head first; then the incoming edges in batches of kAggB whose Wigner rows and
// softmax weights are staged in shared memory; each thread issues all of an edge's
// y loads before its FMAs.  Template parameters fix the kept rows (lmax, mmax).
constexpr int kAggB = 8;
constexpr int kAggWfl = 240;   // >= egnn_wigner_floats(6, 2) = 235

template <int LM, int MM>
__global__ void __launch_bounds__(128) agg_kernel(const __grid_constant__ TcParams P) {
  constexpr int L = LM + 1;
  constexpr int NR = (MM == 0) ? L : (MM == 1 ? 3 * L - 2 : 5 * L - 6);   // kept rows
  __shared__ float Ds[kAggB * kAggWfl];
  __shared__ float ps[kAggB * 16];
  __shared__ float hmx[16], hinv[16];
  const int d = blockIdx.x;
  const int c = threadIdx.x;
  const int C = P.C, H = P.H, hc = P.C / P.H;
  const int h = c / hc;
  int e0 = P.row_ptr[d], e1 = P.row_ptr[d + 1];
  if (e0 < 0 || e1 < e0 || e1 > P.n_edges) {
    if (c == 0) egnn_flag(P.status, EGNN_DEV_BAD_GRAPH);
    e1 = e0;
  }
  float mx = -INFINITY;
  for (int e = e0; e < e1; ++e) mx = fmaxf(mx, P.logits[(long long)e * H + h]);
  float sum = 0.f;
  for (int e = e0; e < e1; ++e) sum += __expf(P.logits[(long long)e * H + h] - mx);
  if (c % hc == 0) {
    hmx[h] = mx;
    hinv[h] = e1 > e0 ? 1.0f / sum : 0.f;
  }
  // column of kept row (l, m) in y, and its Wigner offset, resolved at compile time
  int col[NR], wo[NR], rl[NR];
  {
    int r = 0;
#pragma unroll
    for (int l = 0; l < L; ++l) {
      const int ml = l < MM ? l : MM;
#pragma unroll
      for (int m = -ml; m <= ml; ++m) {
        const int b = m < 0 ? -m : m;
        col[r] = b == 0 ? l * C : P.ybase[b] + (m > 0 ? 0 : (L - b) * C) + (l - b) * C;
        wo[r] = P.woff[l] + (m + ml) * (2 * l + 1);
        rl[r] = l;
        ++r;
      }
    }
  }
  float acc[L * L];
#pragma unroll
  for (int i = 0; i < L * L; ++i) acc[i] = 0.f;
  for (int eb = e0; eb < e1; eb += kAggB) {
    const int nb = min(kAggB, e1 - eb);
    __syncthreads();
    for (int i = c; i < nb * P.wfl; i += 128) Ds[(i / P.wfl) * kAggWfl + i % P.wfl] = P.wig[(long long)eb * P.wfl + i];
    for (int i = c; i < nb * H; i += 128) {
      const int j = i / H, hh = i - j * H;
      ps[j * 16 + hh] = __expf(P.logits[(long long)(eb + j) * H + hh] - hmx[hh]) * hinv[hh];
    }
    __syncthreads();
    for (int j = 0; j < nb; ++j) {
      const __nv_bfloat16* y = P.Y + (long long)(eb + j) * P.ncols_y + c;
      float yv[NR];
#pragma unroll
      for (int r = 0; r < NR; ++r) yv[r] = __bfloat162float(y[col[r]]);
      const float pe = ps[j * 16 + h];
      const float* Dj = Ds + j * kAggWfl;
#pragma unroll
      for (int r = 0; r < NR; ++r) {
        const int l = rl[r];
        const float v = pe * yv[r];
#pragma unroll
        for (int mp = 0; mp < 2 * l + 1; ++mp) acc[l * l + mp] += Dj[wo[r] + mp] * v;
      }
    }
  }
  const long long ob = (long long)d * L * L * C;
#pragma unroll
  for (int i = 0; i < L * L; ++i) {
    float v = __bfloat162float(P.node_in[ob + i * C + c]) + acc[i];
    P.node_out[ob + i * C + c] = __float2bfloat16_rn(v);
  }
}

template <int MM>
cudaError_t launch_agg_mm(const TcParams& P, cudaStream_t st) {
  switch (P.lmax) {
    case 1: if (MM <= 1) agg_kernel<1, (MM <= 1 ? MM : 1)><<<P.n_atoms, 128, 0, st>>>(P); break;
    case 2: agg_kernel<2, MM><<<P.n_atoms, 128, 0, st>>>(P); break;
    case 3: agg_kernel<3, MM><<<P.n_atoms, 128, 0, st>>>(P); break;
    case 4: agg_kernel<4, MM><<<P.n_atoms, 128, 0, st>>>(P); break;
    case 5: agg_kernel<5, MM><<<P.n_atoms, 128, 0, st>>>(P); break;
    default: agg_kernel<6, MM><<<P.n_atoms, 128, 0, st>>>(P); break;
  }
  return cudaGetLastError();
}

// Hamiltonian head from y.  Persistent CTAs stage U^T (all L) in shared memory once,
// then loop over groups of `te` edges: t = rotate-back of y, labels
// h[L][M][k] = sum_c U^L[k][c] t[L, M, c] (lanes run over k: consecutive addresses in
// U^T), block = sum of Clebsch-Gordan images.
__global__ void __launch_bounds__(256) head_blocks_kernel(const __grid_constant__ TcParams P,
                                                          const __grid_constant__ HeadTables Tb, HeadUPtrs Up,
                                                          float* __restrict__ blocks, int te, int u_total) {
  extern __shared__ float hsm[];
  const int C = P.C, L = P.L, L2 = P.L2, mmax = P.mmax;
  const int nlab = Tb.n_lab, norb = Tb.n_orb;
  float* Us = hsm;                        // per L: [C][mult_L] at uoff(L) = C * sum_{L'<L} mult_L'
  float* Ds = Us + u_total;               // [te][wfl]
  float* Ts = Ds + te * P.wfl;            // [te][L2][C]
  float* Ls = Ts + te * L2 * C;           // [te][nlab]
  const int tid = threadIdx.x, nt = blockDim.x;
  {
    int uo = 0;
    for (int Lq = 0; Lq <= P.lmax; ++Lq) {
      const int mult = Tb.mult[Lq];
      for (int i = tid; i < mult * C; i += nt) {
        const int k = i / C, c = i - k * C;
        Us[uo + c * mult + k] = __bfloat162float(Up.U[Lq][i]);
      }
      uo += mult * C;
    }
  }
  const long long ngroups = (P.n_edges + te - 1) / te;
  for (long long gi = blockIdx.x; gi < ngroups; gi += gridDim.x) {
    const long long e0 = gi * te;
    const int ne = (int)min((long long)te, P.n_edges - e0);
    __syncthreads();
    for (int i = tid; i < ne * P.wfl; i += nt) Ds[i] = P.wig[e0 * P.wfl + i];
    __syncthreads();
    for (int i = tid; i < ne * L2 * C; i += nt) {
      const int e = i / (L2 * C), rr = i - e * L2 * C;
      const int lm = rr / C, c = rr - lm * C;
      int l = 0;
      while ((l + 1) * (l + 1) <= lm) ++l;
      const int mp = lm - l * l - l, ml = l < mmax ? l : mmax, dl = 2 * l + 1;
      const float* Dl = Ds + e * P.wfl + P.woff[l];
      const __nv_bfloat16* y = P.Y + (e0 + e) * (long long)P.ncols_y;
      float v = 0.f;
      for (int m = -ml; m <= ml; ++m) {
        const int b = m < 0 ? -m : m;
        const int col = b == 0 ? l * C : P.ybase[b] + (m > 0 ? 0 : (L - b) * C) + (l - b) * C;
        v += Dl[(m + ml) * dl + (mp + l)] * __bfloat162float(y[col + c]);
      }
      Ts[i] = v;
    }
    __syncthreads();
    for (int i = tid; i < ne * nlab; i += nt) {
      const int e = i / nlab, q = i - e * nlab;
      int Lq = 0;
      while (Lq + 1 <= P.lmax && Tb.lab_off[Lq + 1] <= q) ++Lq;
      const int mult = Tb.mult[Lq];
      const int r = q - Tb.lab_off[Lq];
      const int M = r / mult, k = r - M * mult;
      int uo = 0;
      for (int Lp = 0; Lp < Lq; ++Lp) uo += Tb.mult[Lp] * C;
      const float* U = Us + uo + k;
      const float* t = Ts + (e * L2 + Lq * Lq + M) * C;
      float a = 0.f;
#pragma unroll 8
      for (int c = 0; c < C; ++c) a += U[c * mult] * t[c];
      Ls[i] = a;
    }
    __syncthreads();
    for (int i = tid; i < ne * norb * norb; i += nt) {
      const int e = i / (norb * norb), q = i - e * norb * norb;
      const int ri = q / norb, cj = q - ri * norb;
      const int a = Tb.orb_shell[ri], b = Tb.orb_shell[cj];
      const int la = Tb.shell_l[a], lb = Tb.shell_l[b];
      const int ia = ri - Tb.shell_off[a], jb = cj - Tb.shell_off[b];
      float v = 0.f;
      for (int Lc = (la > lb ? la - lb : lb - la); Lc <= la + lb; ++Lc) {
        const int k = Tb.kidx[(a * Tb.n_shells + b) * 8 + Lc];
        const float* cgm = Tb.cg + Tb.cg_off[(la * 4 + lb) * 8 + Lc] + (ia * (2 * lb + 1) + jb) * (2 * Lc + 1);
        const float* h = Ls + e * nlab + Tb.lab_off[Lc] + k;
        const int mult = Tb.mult[Lc];
        for (int M = 0; M < 2 * Lc + 1; ++M) v += cgm[M] * h[M * mult];
      }
      blocks[(e0 + e) * norb * norb + q] = v;
    }
  }
}

}  // namespace

size_t so2_tc_smem_bytes() { return kSA * kAStage + kSB * kBStage + sizeof(SmemCtl) + 1024; }

static cudaError_t launch_tc_gemm(const TcParams& P, const TcWeights& W, cudaStream_t st) {
  long long total = P.wprep_bytes / 2;
  prep_weights_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(P, W.W2, W.W0, W.Wm[0][0], W.Wm[0][1],
                                                                      W.Wm[1][0], W.Wm[1][1], total,
                                                                      const_cast<uint8_t*>(P.wprep));
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (P.n_edges > 0) {
    size_t sm = so2_tc_smem_bytes();
    err = cudaFuncSetAttribute(so2_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (err != cudaSuccess) return err;
    so2_tc_kernel<<<P.grid, kThreads, sm, st>>>(P);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
  }
  return cudaSuccess;
}

size_t head_tc_smem_bytes(const TcParams& P, int n_lab, int te) {
  return sizeof(float) * (size_t)te * (P.wfl + P.L2 * P.C + n_lab);
}

cudaError_t launch_head_tc(const TcParams& P, const TcWeights& W, const HeadTables& T, HeadUPtrs U,
                           float* blocks, cudaStream_t st) {
  cudaError_t err = launch_tc_gemm(P, W, st);
  if (err != cudaSuccess || P.n_edges == 0) return err;
  int u_total = 0;
  for (int Lq = 0; Lq <= P.lmax; ++Lq) u_total += T.mult[Lq] * P.C;
  int te = 16;   // edges per group; aim at two CTAs per SM (<= 110 KB of shared memory each)
  while (te > 1 && sizeof(float) * (size_t)u_total + head_tc_smem_bytes(P, T.n_lab, te) > 110 * 1024) te >>= 1;
  size_t sm = sizeof(float) * (size_t)u_total + head_tc_smem_bytes(P, T.n_lab, te);
  if (sm > 220 * 1024) return cudaErrorInvalidValue;
  err = cudaFuncSetAttribute(head_blocks_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (err != cudaSuccess) return err;
  long long groups = (P.n_edges + te - 1) / te;
  int grid = (int)(groups < 4LL * P.grid ? groups : 4LL * P.grid);
  head_blocks_kernel<<<grid, 256, sm, st>>>(P, T, U, blocks, te, u_total);
  return cudaGetLastError();
}

cudaError_t launch_layer_tc(const TcParams& P, const TcWeights& W, cudaStream_t st) {
  cudaError_t err = launch_tc_gemm(P, W, st);
  if (err != cudaSuccess) return err;
  switch (P.mmax) {
    case 0: return launch_agg_mm<0>(P, st);
    case 1: return launch_agg_mm<1>(P, st);
    default: return launch_agg_mm<2>(P, st);
  }
}
