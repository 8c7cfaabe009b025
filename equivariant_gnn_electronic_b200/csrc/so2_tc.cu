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
//                                -> y_e (bf16).
//                 Warp roles: 0 bulk-copies B tiles, 1 issues MMAs (one thread)
//                 and owns TMEM, 2-5 build A tiles, 6-9 drain TMEM.
//   agg           one CTA per destination atom, thread = channel pair: attention
//                 logits from SiLU(y0), online softmax over the atom's incoming
//                 edges, rotate y back with the kept rows of D^l(R_e), weighted
//                 sum, residual; no atomics.
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

constexpr int kHStage = 2 * kAStage;   // radial hidden layer of a tile, K = 128: 2 chunks

struct SmemCtl {
  uint64_t a_full[kSA], a_empty[kSA], b_full[kSB], b_empty[kSB];
  uint64_t acc_full, acc_empty, gate_ready, mma_done, hid_full, hid_empty;
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

// acc[i] (+)= sum_{mp < dl} co[mp] * z[mp*C + 2i .. 2i+1] for 32 fp16 channels held as
// 16 half2, in packed fp16 arithmetic (one HFMA2 per channel pair and row); three rows
// of z (12 x 16 B) are loaded before their FMAs.
__device__ __forceinline__ void rot_h1(__half2* acc, const __half* z, int C, const float* co, int dl) {
  for (int mp0 = 0; mp0 < dl; mp0 += 3) {
    uint4 q[3][4];
    __half2 c[3];
#pragma unroll
    for (int u = 0; u < 3; ++u) {
      const bool ok = mp0 + u < dl;
      const uint4* zp = reinterpret_cast<const uint4*>(z + (ok ? mp0 + u : 0) * C);
#pragma unroll
      for (int k = 0; k < 4; ++k) q[u][k] = ok ? __ldg(zp + k) : make_uint4(0, 0, 0, 0);
      c[u] = __float2half2_rn(ok ? __ldg(co + mp0 + u) : 0.f);
    }
#pragma unroll
    for (int u = 0; u < 3; ++u)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __half2* h = reinterpret_cast<const __half2*>(&q[u][k]);
#pragma unroll
        for (int i = 0; i < 4; ++i) acc[4 * k + i] = __hfma2(c[u], h[i], acc[4 * k + i]);
      }
  }
}

// Same for two coefficient rows at once (the +b and -b rows share z), two rows of z
// (8 x 16 B) in flight per batch.
__device__ __forceinline__ void rot_h2(__half2* ap, __half2* am, const __half* z, int C, const float* cop,
                                       const float* com, int dl) {
  for (int mp0 = 0; mp0 < dl; mp0 += 2) {
    uint4 q[2][4];
    __half2 cp[2], cm[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const bool ok = mp0 + u < dl;
      const uint4* zp = reinterpret_cast<const uint4*>(z + (ok ? mp0 + u : 0) * C);
#pragma unroll
      for (int k = 0; k < 4; ++k) q[u][k] = ok ? __ldg(zp + k) : make_uint4(0, 0, 0, 0);
      cp[u] = __float2half2_rn(ok ? __ldg(cop + mp0 + u) : 0.f);
      cm[u] = __float2half2_rn(ok ? __ldg(com + mp0 + u) : 0.f);
    }
#pragma unroll
    for (int u = 0; u < 2; ++u)
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const __half2* h = reinterpret_cast<const __half2*>(&q[u][k]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ap[4 * k + i] = __hfma2(cp[u], h[i], ap[4 * k + i]);
          am[4 * k + i] = __hfma2(cm[u], h[i], am[4 * k + i]);
        }
      }
  }
}

// acc[i] *= g[i] for 32 fp16 channels (16 half2) read from the gate scratch.
__device__ __forceinline__ void gate_mul(__half2* acc, const __half* g) {
  const uint4* gp = reinterpret_cast<const uint4*>(g);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint4 w = gp[k];
    const __half2* h = reinterpret_cast<const __half2*>(&w);
#pragma unroll
    for (int i = 0; i < 4; ++i) acc[4 * k + i] = __hmul2(acc[4 * k + i], h[i]);
  }
}

// Writes 32 fp16 values (16 half2) as columns [32*half, 32*half+32) of row r of a
// 128B-swizzled K-major tile.
__device__ __forceinline__ void store_row_h(uint8_t* tile, int r, int half, const __half2* v) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int chunk = half * 4 + q;
    uint4 w;
    w.x = *reinterpret_cast<const uint32_t*>(&v[4 * q + 0]);
    w.y = *reinterpret_cast<const uint32_t*>(&v[4 * q + 1]);
    w.z = *reinterpret_cast<const uint32_t*>(&v[4 * q + 2]);
    w.w = *reinterpret_cast<const uint32_t*>(&v[4 * q + 3]);
    *reinterpret_cast<uint4*>(tile + r * 128 + ((chunk ^ (r & 7)) << 4)) = w;
  }
}

__device__ __forceinline__ uint32_t pack2h(float a, float b) {
  __half2 h = __floats2half2_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// Writes 32 fp32 values, rounded to fp16, as columns [32*half, 32*half+32) of row r
// of a 128B-swizzled K-major tile.
__device__ __forceinline__ void store_row32(uint8_t* tile, int r, int half, const float* v) {
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    int chunk = half * 4 + q;
    uint4 w;
    w.x = pack2h(v[8 * q + 0], v[8 * q + 1]);
    w.y = pack2h(v[8 * q + 2], v[8 * q + 3]);
    w.z = pack2h(v[8 * q + 4], v[8 * q + 5]);
    w.w = pack2h(v[8 * q + 6], v[8 * q + 7]);
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
  uint8_t* Hbuf = Bbuf + kSB * kBStage;
  SmemCtl* ctl = reinterpret_cast<SmemCtl*>(Hbuf + kHStage);
  const uint32_t A_u32 = base_u32;
  const uint32_t B_u32 = base_u32 + kSA * kAStage;
  const uint32_t H_u32 = B_u32 + kSB * kBStage;
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
    tc::mbar_init(tc::smem_u32(&ctl->hid_full), kProducers);
    tc::mbar_init(tc::smem_u32(&ctl->hid_empty), 1);
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
  const int C = P.C, K = P.K;
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
            if (!tc::mbar_wait(tc::smem_u32(&ctl->b_empty[sb]), ((ib / kSB) & 1) ^ 1, P.status, abort, 64)) break;
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
      uint32_t ia = 0, ib = 0, ip = 0, it = 0;
      for (int t = blockIdx.x; t < P.n_tiles && !*abort; t += gridDim.x, ++it) {
        bool hid_waited = false;
        for (int p = 0; p < P.npass && !*abort; ++p, ++ip) {
          const TcPass& ps = P.pass[p];
          if (!tc::mbar_wait(tc::smem_u32(&ctl->acc_empty), (ip & 1) ^ 1, P.status, abort, 32)) break;
          if (ps.kind == 0 && !hid_waited) {
            if (!tc::mbar_wait(tc::smem_u32(&ctl->hid_full), it & 1, P.status, abort, 32)) break;
            hid_waited = true;
          }
          tc::tc_fence_after();
          for (int j = 0; j < ps.nk; ++j, ++ib) {
            const int sb = ib % kSB;
            int sa = 0;
            uint32_t a_base;
            if (ps.kind == 0) {
              a_base = H_u32 + j * kAStage;           // hidden layer, resident for the whole tile
            } else {
              sa = ia % kSA;
              if (!tc::mbar_wait(tc::smem_u32(&ctl->a_full[sa]), (ia / kSA) & 1, P.status, abort, 32)) break;
              a_base = A_u32 + sa * kAStage;
            }
            if (!tc::mbar_wait(tc::smem_u32(&ctl->b_full[sb]), (ib / kSB) & 1, P.status, abort, 32)) break;
            tc::tc_fence_after();
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              uint64_t ad = tc::sw128_desc(a_base + ks * 32);
              for (int n0 = 0; n0 < ps.n; n0 += 256) {
                int ns = ps.n - n0 < 256 ? ps.n - n0 : 256;
                uint64_t bd = tc::sw128_desc(B_u32 + sb * kBStage + n0 * 128 + ks * 32);
                tc::mma_bf16(tmem + n0, ad, bd, tc::idesc_f16(128, ns), (j > 0 || ks > 0) ? 1u : 0u);
              }
            }
            if (ps.kind != 0) {
              tc::mma_commit(tc::smem_u32(&ctl->a_empty[sa]));
              ++ia;
            }
            tc::mma_commit(tc::smem_u32(&ctl->b_empty[sb]));
          }
          if (ps.kind == 0 && ps.last_of_kind) tc::mma_commit(tc::smem_u32(&ctl->hid_empty));
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
    const __half* gsc = P.gate_scratch + ((long long)blockIdx.x * 128 + r) * P.gcols;
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
      // radial hidden layer SiLU(W1 rho(|r_e|) + b1), once per tile, into Hbuf
      if (!tc::mbar_wait(tc::smem_u32(&ctl->hid_empty), (it & 1) ^ 1, P.status, abort, 64)) break;
      {
        const float mu_step = P.rcut / (float)(K - 1);
        const float inv2s2 = 1.0f / (2.0f * mu_step * mu_step);
        for (int j = 0; j < C / 64; ++j) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.f;
          if (valid) {
            const int c0 = j * 64 + half * 32;
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = __bfloat162float(P.b1[c0 + i]);
            for (int k0 = 0; k0 < K; k0 += 8) {
              float rho[8];
#pragma unroll
              for (int u = 0; u < 8; ++u) {
                const float dd = dist - (k0 + u) * mu_step;
                rho[u] = (k0 + u < K) ? __expf(-dd * dd * inv2s2) : 0.f;
              }
#pragma unroll 4
              for (int i = 0; i < 32; ++i) {
                // W1 row (c0 + i), columns k0..k0+7 (K is a multiple of 8 or padded by the bound)
                const __nv_bfloat16* wr = P.W1 + (c0 + i) * K + k0;
                float a = 0.f;
#pragma unroll
                for (int u = 0; u < 8; ++u)
                  if (k0 + u < K) a += __bfloat162float(wr[u]) * rho[u];
                v[i] += a;
              }
            }
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = v[i] / (1.0f + __expf(-v[i]));
          }
          store_row32(Hbuf + j * kAStage, r, half, v);
        }
        tc::fence_proxy_async_smem();
        tc::mbar_arrive(tc::smem_u32(&ctl->hid_full));
      }
      bool gate_waited = false;
      for (int p = 0; p < P.npass && !*abort; ++p) {
        const TcPass& ps = P.pass[p];
        if (ps.kind == 0) continue;
        if (!gate_waited) {
          if (!tc::mbar_wait(tc::smem_u32(&ctl->gate_ready), it & 1, P.status, abort, 64)) break;
          gate_waited = true;
        }
        const int b = ps.block;
        if (b == 0) {
          for (int j = 0; j < ps.nk; ++j, ++ia) {
            int sa = ia % kSA;
            if (!tc::mbar_wait(tc::smem_u32(&ctl->a_empty[sa]), ((ia / kSA) & 1) ^ 1, P.status, abort, 32)) break;
            uint8_t* tile = Abuf + sa * kAStage;
            const int l = j / (C2 / 64), c2b = j % (C2 / 64);
            const int dl = 2 * l + 1, ml = l < P.mmax ? l : P.mmax;
            const float* Drow = De + P.woff[l] + ml * dl;          // row m = 0
            const int cs = c2b * 64;
            const __half* z = (cs < C) ? P.node_h + ((long long)s * P.L2 + l * l) * C + cs
                                       : P.node_h + ((long long)d * P.L2 + l * l) * C + (cs - C);
            {
              __half2 acc[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) acc[i] = __float2half2_rn(0.f);
              if (valid) {
                rot_h1(acc, z + half * 32, C, Drow, dl);
                gate_mul(acc, gsc + l * C2 + cs + half * 32);
              }
              store_row_h(tile, r, half, acc);
            }
            tc::fence_proxy_async_smem();
            tc::mbar_arrive(tc::smem_u32(&ctl->a_full[sa]));
          }
        } else {
          // chunk pairs (+b, -b) of the same (l, 64 channels): z is read once for both
          for (int j = 0; j < ps.nk; j += 2, ia += 2) {
            int sa0 = ia % kSA, sa1 = (ia + 1) % kSA;
            if (!tc::mbar_wait(tc::smem_u32(&ctl->a_empty[sa0]), ((ia / kSA) & 1) ^ 1, P.status, abort, 32)) break;
            if (!tc::mbar_wait(tc::smem_u32(&ctl->a_empty[sa1]), (((ia + 1) / kSA) & 1) ^ 1, P.status, abort, 32))
              break;
            uint8_t* tp = Abuf + sa0 * kAStage;
            uint8_t* tm = Abuf + sa1 * kAStage;
            const int q2 = j >> 1;
            const int l = b + q2 / (C2 / 64), c2b = q2 % (C2 / 64);
            const int dl = 2 * l + 1, ml = l < P.mmax ? l : P.mmax;
            const float* Dp = De + P.woff[l] + (ml + b) * dl;
            const float* Dm = De + P.woff[l] + (ml - b) * dl;
            const int cs = c2b * 64;
            const __half* z = (cs < C) ? P.node_h + ((long long)s * P.L2 + l * l) * C + cs
                                       : P.node_h + ((long long)d * P.L2 + l * l) * C + (cs - C);
            {
              __half2 ap[16], am[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) ap[i] = am[i] = __float2half2_rn(0.f);
              if (valid) {
                rot_h2(ap, am, z + half * 32, C, Dp, Dm, dl);
                gate_mul(ap, gsc + l * C2 + cs + half * 32);
                gate_mul(am, gsc + l * C2 + cs + half * 32);
              }
              store_row_h(tp, r, half, ap);
              store_row_h(tm, r, half, am);
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
    __half* gsc = P.gate_scratch + ((long long)blockIdx.x * 128 + r) * P.gcols;
    uint32_t ip = 0;
    const int H = P.H;
    for (int t = blockIdx.x; t < P.n_tiles && !*abort; t += gridDim.x) {
      const long long e = (long long)t * 128 + r;
      const bool valid = e < E;
      float lg[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) lg[h] = 0.f;
      for (int p = 0; p < P.npass && !*abort; ++p, ++ip) {
        const TcPass& ps = P.pass[p];
        if (!tc::mbar_wait(tc::smem_u32(&ctl->acc_full), ip & 1, P.status, abort, 256)) break;
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
              dst[q] = make_uint4(pack2h(v[8 * q], v[8 * q + 1]), pack2h(v[8 * q + 2], v[8 * q + 3]),
                                  pack2h(v[8 * q + 4], v[8 * q + 5]), pack2h(v[8 * q + 6], v[8 * q + 7]));
          } else if (valid) {
            uint8_t* yrow = P.Y + e * (long long)P.y_row_bytes;
            if (ps.block == 0) {               // y0 stays fp32
              uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<float*>(yrow) + col);
#pragma unroll
              for (int q = 0; q < 8; ++q)
                dst[q] = make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]),
                                    __float_as_uint(v[4 * q + 2]), __float_as_uint(v[4 * q + 3]));
              if (P.with_logits) {             // a_h += A[h, col..col+31] . SiLU(y0[col..col+31])
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = v[i] / (1.0f + __expf(-v[i]));
#pragma unroll
                for (int h = 0; h < 16; ++h) {
                  if (h < H) {
                    const float4* Ah = reinterpret_cast<const float4*>(P.Af + (long long)h * P.L * P.C + col);
                    float a = 0.f;
#pragma unroll
                    for (int q = 0; q < 8; ++q) {
                      const float4 w4 = __ldg(Ah + q);
                      a += w4.x * v[4 * q] + w4.y * v[4 * q + 1] + w4.z * v[4 * q + 2] + w4.w * v[4 * q + 3];
                    }
                    lg[h] += a;
                  }
                }
              }
            } else {
              uint4* dst = reinterpret_cast<uint4*>(reinterpret_cast<__nv_bfloat16*>(yrow + P.y0_bytes) +
                                                    (P.ybase[ps.block] - P.ybase[1]) + col);
#pragma unroll
              for (int q = 0; q < 4; ++q)
                dst[q] = make_uint4(pack2(v[8 * q], v[8 * q + 1]), pack2(v[8 * q + 2], v[8 * q + 3]),
                                    pack2(v[8 * q + 4], v[8 * q + 5]), pack2(v[8 * q + 6], v[8 * q + 7]));
            }
          }
        }
        tc::tc_fence_before();
        tc::mbar_arrive(tc::smem_u32(&ctl->acc_empty));
        if (ps.kind == 0 && ps.last_of_kind) tc::mbar_arrive(tc::smem_u32(&ctl->gate_ready));
        if (ps.kind == 1 && ps.block == 0 && ps.last_of_kind && valid && P.with_logits) {
#pragma unroll
          for (int h = 0; h < 16; ++h)
            if (h < H) P.logits[e * H + h] = lg[h] + __bfloat162float(P.bA[h]);
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
  reinterpret_cast<__half*>(out)[idx] = __float2half_rn(v);   // bf16 values are exact in fp16
}

// Compile-time layout of kept row r = (l, m) (rows ordered by l, then m = -min(l,MM)..):
// its degree, its padded offset among an edge's staged Wigner rows, and (C = 128) its
// column in y: inside the fp32 y0 section for m = 0, inside the bf16 section otherwise.
template <int MM>
__host__ __device__ constexpr int agg_row_l(int r) {
  int l = 0;
  while (r >= 2 * (l < MM ? l : MM) + 1) { r -= 2 * (l < MM ? l : MM) + 1; ++l; }
  return l;
}
template <int MM>
__host__ __device__ constexpr int agg_row_m(int r) {
  int l = 0;
  while (r >= 2 * (l < MM ? l : MM) + 1) { r -= 2 * (l < MM ? l : MM) + 1; ++l; }
  return r - (l < MM ? l : MM);
}
template <int MM>
__host__ __device__ constexpr int agg_po(int r) {
  int o = 0;
  for (int q = 0; q < r; ++q) o += ((2 * agg_row_l<MM>(q) + 1) + 3) & ~3;
  return o;
}
template <int L, int MM>
__host__ __device__ constexpr int agg_col(int r) {
  const int l = agg_row_l<MM>(r);
  const int ml = l < MM ? l : MM;
  int rr = r;
  for (int q = 0; q < l; ++q) rr -= 2 * (q < MM ? q : MM) + 1;
  const int m = rr - ml;
  const int b = m < 0 ? -m : m;
  const int base16 = b <= 1 ? 0 : 2 * (L - 1) * 128;   // |m| = b block inside the bf16 section
  return b == 0 ? l * 128 : base16 + (m > 0 ? 0 : (L - b) * 128) + (l - b) * 128;
}

// Aggregation: one CTA of 128 threads per destination atom, thread = channel.
// Softmax statistics per head from the logits the SO(2) kernel wrote; then the
// incoming edges in batches of kAggB whose Wigner rows and softmax weights are
// staged in shared memory (one flat, fully parallel copy); per edge all y loads of
// the thread's channel are issued before the FMAs.  No atomics: one owner per atom.
constexpr int kAggB = 8;
constexpr int kAggWfl = 236;   // >= egnn_wigner_floats(6, 2) = 235

template <int MM>
__host__ __device__ constexpr int agg_wo(int r) {   // Wigner float offset of kept row r
  int o = 0;
  for (int q = 0; q < r; ++q) o += 2 * agg_row_l<MM>(q) + 1;
  return o;
}

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
  float acc[L * L];
#pragma unroll
  for (int i = 0; i < L * L; ++i) acc[i] = 0.f;
  for (int eb = e0; eb < e1; eb += kAggB) {
    const int nb = min(kAggB, e1 - eb);
    __syncthreads();
    for (int i = c; i < nb * P.wfl; i += 128) {
      const int j = i / P.wfl;
      Ds[j * kAggWfl + (i - j * P.wfl)] = P.wig[(long long)eb * P.wfl + i];
    }
    for (int i = c; i < nb * H; i += 128) {
      const int j = i / H, hh = i - j * H;
      ps[j * 16 + hh] = __expf(P.logits[(long long)(eb + j) * H + hh] - hmx[hh]) * hinv[hh];
    }
    __syncthreads();
    for (int j = 0; j < nb; ++j) {
      const uint8_t* yrow = P.Y + (long long)(eb + j) * P.y_row_bytes;
      const float* y32 = reinterpret_cast<const float*>(yrow) + c;
      const __nv_bfloat16* y16 = reinterpret_cast<const __nv_bfloat16*>(yrow + P.y0_bytes) + c;
      float yv[NR];
      {
        int r = 0, c16 = 0;
#pragma unroll
        for (int l = 0; l < L; ++l) {
          const int ml = l < MM ? l : MM;
#pragma unroll
          for (int m = -ml; m <= ml; ++m, ++r) {
            if (m == 0) {
              yv[r] = y32[l * 128];
            } else {
              const int b = m < 0 ? -m : m;
              const int col = (b == 1 ? 0 : 2 * (L - 1) * 128) + (m > 0 ? 0 : (L - b) * 128) + (l - b) * 128;
              yv[r] = __bfloat162float(y16[col]);
            }
          }
        }
        (void)c16;
      }
      const float pe = ps[j * 16 + h];
      const float* Dj = Ds + j * kAggWfl;
      {
        int r = 0, wo = 0;
#pragma unroll
        for (int l = 0; l < L; ++l) {
          const int ml = l < MM ? l : MM;
#pragma unroll
          for (int m = -ml; m <= ml; ++m, ++r) {
            const float v = pe * yv[r];
#pragma unroll
            for (int mp = 0; mp < 2 * l + 1; ++mp) acc[l * l + mp] += Dj[wo + mp] * v;
            wo += 2 * l + 1;
          }
        }
      }
    }
  }
  const long long ob = (long long)d * L * L * C;
#pragma unroll
  for (int i = 0; i < L * L; ++i) {
    const float v = __bfloat162float(P.node_in[ob + i * C + c]) + acc[i];
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
template <int LM, int MM>
__global__ void __launch_bounds__(128) head_blocks_kernel(const __grid_constant__ TcParams P,
                                                          const __grid_constant__ HeadTables Tb, HeadUPtrs Up,
                                                          float* __restrict__ blocks, int te, int u_total) {
  extern __shared__ float hsm[];
  const int C = P.C, L2 = P.L2;
  const int nlab = Tb.n_lab, norb = Tb.n_orb;
  int nlk = 0;
  for (int Lq = 0; Lq <= P.lmax; ++Lq) nlk += Tb.mult[Lq];
  float* Us = hsm;                        // per L: [C][mult_L] at uoff(L) = C * sum_{L'<L} mult_L'
  float* Ds = Us + u_total;               // [te][wfl]  (u_total is a multiple of C)
  float* Ts = Ds + ((te * P.wfl + 3) & ~3);   // [te][L2][C], 16-byte aligned for float4 reads
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
    // rotate back: thread = channel; every index below is a compile-time constant
    for (int e = 0; e < ne; ++e) {
      const uint8_t* yrow = P.Y + (e0 + e) * (long long)P.y_row_bytes;
      const float* y32 = reinterpret_cast<const float*>(yrow) + tid;
      const __nv_bfloat16* y16 = reinterpret_cast<const __nv_bfloat16*>(yrow + P.y0_bytes) + tid;
      const float* De = Ds + e * P.wfl;
      float* Te = Ts + (e * L2) * C + tid;
      int wo = 0;
#pragma unroll
      for (int l = 0; l <= LM; ++l) {
        const int ml = l < MM ? l : MM;
        float yv[5];
#pragma unroll
        for (int m = -ml; m <= ml; ++m) {
          const int b = m < 0 ? -m : m;
          yv[m + ml] = b == 0 ? y32[l * 128]
                              : __bfloat162float(y16[(b == 1 ? 0 : 2 * LM * 128) + (m > 0 ? 0 : (LM + 1 - b) * 128) +
                                                     (l - b) * 128]);
        }
        float tv[2 * LM + 1];
#pragma unroll
        for (int mp = 0; mp < 2 * l + 1; ++mp) tv[mp] = 0.f;
#pragma unroll
        for (int m = -ml; m <= ml; ++m)
#pragma unroll
          for (int mp = 0; mp < 2 * l + 1; ++mp) tv[mp] += De[wo + (m + ml) * (2 * l + 1) + mp] * yv[m + ml];
#pragma unroll
        for (int mp = 0; mp < 2 * l + 1; ++mp) Te[(l * l + mp) * C] = tv[mp];
        wo += (2 * ml + 1) * (2 * l + 1);
      }
    }
    // labels: one thread per (edge, L, k) computes every M, so t reads are broadcasts
    // within a warp and U^T reads are consecutive
    for (int i = tid; i < ne * nlk; i += nt) {
      const int e = i / nlk;
      int q = i - e * nlk;
      int Lq = 0, uo = 0;
      while (q >= Tb.mult[Lq]) {
        q -= Tb.mult[Lq];
        uo += Tb.mult[Lq] * C;
        ++Lq;
      }
      const int k = q, mult = Tb.mult[Lq], nM = 2 * Lq + 1;
      const float* U = Us + uo + k;
      const float* t0 = Ts + (e * L2 + Lq * Lq) * C;
      float a[13];
#pragma unroll
      for (int M = 0; M < 13; ++M) a[M] = 0.f;
      for (int c = 0; c < C; c += 4) {
        const float u0 = U[(c + 0) * mult], u1 = U[(c + 1) * mult], u2 = U[(c + 2) * mult], u3 = U[(c + 3) * mult];
#pragma unroll
        for (int M = 0; M < 13; ++M) {
          if (M < nM) {
            const float4 tv = *reinterpret_cast<const float4*>(t0 + M * C + c);
            a[M] += u0 * tv.x + u1 * tv.y + u2 * tv.z + u3 * tv.w;
          }
        }
      }
      float* out = Ls + e * nlab + Tb.lab_off[Lq] + k;
#pragma unroll
      for (int M = 0; M < 13; ++M)
        if (M < nM) out[M * mult] = a[M];
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

size_t so2_tc_smem_bytes() { return kSA * kAStage + kSB * kBStage + kHStage + sizeof(SmemCtl) + 1024; }

// bf16 -> fp16 copy of the node table (exact for the embeddings' range), 8 values per thread.
__global__ void to_f16_kernel(const __nv_bfloat16* __restrict__ in, __half* __restrict__ out, long long n8) {
  long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n8) return;
  const uint4 q = reinterpret_cast<const uint4*>(in)[i];
  float f[8];
  unpack8(q, f);
  uint4 o;
  o.x = pack2h(f[0], f[1]);
  o.y = pack2h(f[2], f[3]);
  o.z = pack2h(f[4], f[5]);
  o.w = pack2h(f[6], f[7]);
  reinterpret_cast<uint4*>(out)[i] = o;
}

__global__ void a_to_f32_kernel(const __nv_bfloat16* __restrict__ A, float* __restrict__ out, int n) {
  int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) out[i] = __bfloat162float(A[i]);
}

static cudaError_t launch_tc_gemm(const TcParams& P, const TcWeights& W, cudaStream_t st) {
  if (P.with_logits) {
    const int na = P.H * P.L * P.C;
    a_to_f32_kernel<<<(na + 255) / 256, 256, 0, st>>>(P.A, P.Af, na);
  }
  const long long n8 = (long long)P.n_atoms * P.L2 * P.C / 8;
  to_f16_kernel<<<(unsigned)((n8 + 255) / 256), 256, 0, st>>>(P.node_in, P.node_h, n8);
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
  return sizeof(float) * ((size_t)((te * P.wfl + 3) & ~3) + (size_t)te * (P.L2 * P.C + n_lab));
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
  long long groups = (P.n_edges + te - 1) / te;
  int grid = (int)(groups < 4LL * P.grid ? groups : 4LL * P.grid);
  switch (P.mmax * 8 + P.lmax) {
#define EGNN_HEAD_CASE(LMv, MMv)                                                                      \
  case MMv * 8 + LMv:                                                                                \
    err = cudaFuncSetAttribute(head_blocks_kernel<LMv, MMv>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm); \
    if (err != cudaSuccess) return err;                                                              \
    head_blocks_kernel<LMv, MMv><<<grid, 128, sm, st>>>(P, T, U, blocks, te, u_total);                \
    break;
    EGNN_HEAD_CASE(1, 0) EGNN_HEAD_CASE(2, 0) EGNN_HEAD_CASE(3, 0) EGNN_HEAD_CASE(4, 0) EGNN_HEAD_CASE(5, 0)
    EGNN_HEAD_CASE(6, 0) EGNN_HEAD_CASE(1, 1) EGNN_HEAD_CASE(2, 1) EGNN_HEAD_CASE(3, 1) EGNN_HEAD_CASE(4, 1)
    EGNN_HEAD_CASE(5, 1) EGNN_HEAD_CASE(6, 1) EGNN_HEAD_CASE(2, 2) EGNN_HEAD_CASE(3, 2) EGNN_HEAD_CASE(4, 2)
    EGNN_HEAD_CASE(5, 2) EGNN_HEAD_CASE(6, 2)
#undef EGNN_HEAD_CASE
    default:
      return cudaErrorInvalidValue;
  }
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
