// Launch parameters of the tensor-core eSCN layer (CUDA path only).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

// One GEMM pass over a 128-edge tile: D[128 x n] = A[128 x 64*nk] B[n x 64*nk]^T, n <= 256
// so that two accumulators alternate in TMEM.  For a block with |m| = b > 0 the pass
// covers output rows [n_off, n_off + np) of both y+ and y- (n = 2 np) and B holds only
// the rows of W_b1 and W_b2 (the sign comes from the instruction's negate-B bit).
struct TcPass {
  int kind;          // 0 = radial gate (A = hidden layer), 1 = SO(2) block
  int block;         // |m| of the SO(2) block
  int n;             // accumulator columns (<= 256, multiple of 32)
  int n_off;         // first output row of the block matrix covered by this pass
  int nk;            // K chunks of 64
  int last_of_kind;  // last gate pass / last pass of block 0
  int np;            // |m| > 0 blocks: output rows per half; accumulator = [y+ rows | y- rows]
  long long boff;    // byte offset of the pass's first B tile in the prepared image
  int roff;          // label mode: float offset of the pass's columns in an edge's record
};

struct TcParams {
  int n_atoms;
  long long n_edges;
  int n_tiles, grid;
  int lmax, mmax, C, H, K, L, L2, wfl, ncols_y, gcols;
  int y_row_bytes;   // bytes of one edge's y record: y0 in fp32, then the |m| > 0 blocks in bf16
  int y0_bytes;      // L * C * 4
  float rcut;
  const int32_t* row_ptr;
  const int32_t* src;
  const float* dist;
  const float* wig;
  const __nv_bfloat16* node_in;
  __nv_bfloat16* node_out;
  const __nv_bfloat16 *W1, *b1, *b2, *A, *bA;
  const uint8_t* wprep;
  long long wprep_bytes;
  uint8_t* Y;                    // head: [n_edges][y_row_bytes]
  int32_t* status;
  // Label mode (head only): the SO(2) weights are pre-multiplied by the label maps U^L,
  // so a pass produces labels in the edge frame, s[l, m, k] = sum_c U^l[k, c] y[l, m, c],
  // stored in fp32 as the concatenation of the passes' accumulators (record of
  // y_row_bytes = 4 * sum of pass widths).
  int label_mode;
  int hroff[3];                  // record offset of block b's first pass
  int hnr[3];                    // label rows of block b: sum_{l >= b} mult_l
  int mult[8];                   // labels per L
  const __nv_bfloat16* U[8];     // U^L [mult_L][C]
  // Tile range of one launch and the per-range buffer of the pipeline (gate + rotate ->
  // SO(2) GEMM): the rotated, gated A operands as 128 x 64 bf16 tiles in the 128-byte-swizzled
  // K-major image the MMA reads, `nch` tiles per edge tile, block b's first at
  // xbase[b] (a |m| > 0 K block stores x+ then x-).
  int t_begin, t_end;
  uint8_t* X;                    // [(t_end - t_begin)][nch][128 * 128 B]
  int nch;
  int xbase[3];
  // Fused layer (layer_fused_kernel): per-CTA stash of y0 in bf16, [grid][L][128][C];
  // per-atom fp32 accumulators of the destinations whose incoming edges lie inside one
  // edge tile, [n_atoms][L^2][C]; and two partial records per edge tile for the
  // destinations whose edges cross a tile boundary, [n_tiles][2][rec_floats], a record
  // being the unnormalised weighted sum [L^2][C], then the per-head softmax maximum [16]
  // and denominator [16] of the tile's part of the segment.
  __nv_bfloat16* stash;
  int32_t* edge_dst;             // destination atom of every edge (fused layer)
  float* acc_g;
  float* slots;
  int rec_floats;
  int own_b;                     // bit l set: the fused layer's second epilogue group owns degree l
  int f_nxs, f_nws, f_dgroup;    // fused layer: x and weight stages, floats of its work buffer per group
  int npass;
  TcPass pass[32];
  int woff[8];
  int ybase[3];
};

struct TcWeights {
  const __nv_bfloat16 *W2, *W0;
  const __nv_bfloat16* Wm[2][2];
};

constexpr int kTcMaxGrid = 160;

// SO(2) GEMM pass width in TMEM columns: 512 = one accumulator per pass (fewer A
// re-reads, drain between passes), 256 = two alternating accumulators (drain overlaps
// the next pass).
#ifndef EGNN_ACC_COLS
#define EGNN_ACC_COLS 256
#endif
constexpr int kTcAccCols = EGNN_ACC_COLS;
constexpr int kTcPairRows = kTcAccCols / 2;   // label / output rows per half of a |m| > 0 pass
constexpr int kTcChunkTiles = 4096;   // edge tiles per launch range (bounds the gate and A buffers)

// Tiles per launch range: the fewest ranges of at most kTcChunkTiles, balanced.
inline int tc_chunk_tiles(int n_tiles) {
  if (n_tiles <= 0) return 1;
  const int nr = (n_tiles + kTcChunkTiles - 1) / kTcChunkTiles;
  return (n_tiles + nr - 1) / nr;
}

struct HeadTables;
struct HeadUPtrs {
  const __nv_bfloat16* U[8];
};
// Precomputed tables of the label-mode head (device memory, built on the host):
// lab[q][11]: number of terms, then up to five Wigner offsets and five record offsets
// of label q's rotate-back; term_ptr[n_orb^2 + 1] / term[]: per block entry its terms
// (label index, Clebsch-Gordan coefficient as float bits).
struct HeadLabelTabs {
  int n_lab, n_orb, n_term;
  const int* lab;
  const int* term_ptr;
  const int2* term;
};

// Consumer of one range's A tiles: launches its kernel over tiles [Ps.t_begin, Ps.t_end).
using TcConsumer = cudaError_t (*)(const TcParams& Ps, int grid, cudaStream_t st, void* ctx);
cudaError_t launch_tc_pipeline(const TcParams& P, const TcWeights& W, cudaStream_t st, TcConsumer consumer,
                               void* ctx, bool profiled);
cudaError_t launch_layer_fused(const TcParams& P, const TcWeights& W, cudaStream_t st);
cudaError_t launch_head_tc(const TcParams& P, const TcWeights& W, const HeadTables& T, HeadUPtrs U,
                           const HeadLabelTabs& LT, float* blocks, cudaStream_t st);
size_t head_tc_smem_bytes(const TcParams& P, int n_lab, int te);
void tc_profile_enable(bool on);
cudaError_t launch_wait_check(int32_t* status, unsigned long long limit_ns, cudaStream_t st);
cudaError_t tc_profile_read(double* ms, long long* launches, long long* edges);
