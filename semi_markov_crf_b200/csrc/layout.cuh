// layout.cuh -- sizes, launch geometry and workspace layout shared by the
// host layer and the kernels.
#pragma once

#include <cstddef>
#include <cstdint>
#include <vector_types.h>

namespace semicrf {

constexpr int C_MAX = 128;
constexpr int K_MAX = 8192;      // long durations (K > LOG_K_MAX) need C <= 8 ...
constexpr int KC_MAX = 65536;    // ... and run on the pipelined kernels only
constexpr int LOG_K_MAX = 2048;  // largest K of the log-domain kernels' shapes
constexpr int LOG_KC_MAX = 16384;
constexpr int NT_MAX = 512;  // threads per CTA
constexpr int TS = 32;       // prefix-sum rows per TMA tile
constexpr int FLUSH_EVERY = 64;  // positions between fp32 -> fp64 partial flushes
constexpr int PATH_ROWS = 256;  // positions per CTA of the path-score pass (one per thread)

// Problem sizes and the lane mapping chosen for them.
//
// Lane groups of GB lanes (a power of two <= 32) own one label each, for both
// fan-ins: in the k fan-in lane j owns KBT consecutive durations, in the label
// fan-in CAT consecutive labels of the other side.  KBT and CAT are
// compile-time shapes of the kernel instantiation; GA == GB.
struct Dims {
  int B, T, C, K;
  int delta;     // checkpoint spacing ceil(sqrt(T*K))
  int nck;       // checkpoint segments per sequence, ceil(T / delta)
  int Tstride;   // rows per sequence in the prefix-sum arrays (>= T+1, multiple of TS)
  int KBT, GB;   // durations per lane, lanes per label (k fan-in); KBT = 0: no
                 // log-domain shape (long durations), see logok
  int CAT, GA;   // labels per lane, lanes per output label (label fan-in)
  int RL;        // ring entries per label: K + KBT (the first KBT slots are mirrored)
  int PC;        // padded length of the exp-domain label vector (>= GA * CAT)
  int NT;        // threads per CTA of the recursion kernels
  int LB;        // launch bound of the instantiation (256 or 512 threads)
  int prefR;     // rows per prefix-sum chunk
  int nchunk;    // prefix-sum chunks per sequence
  int store_w;   // floats per position in the segment recompute store (2C + 2)
  int store_smem;  // 1: the recompute store lives in shared memory
  // Pipelined exponential-domain rings (chain_exp.cu): xG combine lanes per
  // label with xCAT weights each, xH helper lanes per label with xKBH
  // durations each (k = 3..K), xNT threads (launch bound xLB), ring of
  // xRL = K + xKBH entries per label, label vector padded to xPC = xG * xCAT.
  int xG, xCAT, xH, xKBH, xNT, xLB, xRL, xPC;
  // Thread-block cluster of the pipelined rings: xN CTAs per ring (1: one
  // CTA), each owning xCr = ceil(C / xN) consecutive labels; the label
  // vector is exchanged through distributed shared memory every step.
  int xN, xCr;
  // Pipelined Viterbi (viterbi_pipe.cu): helper lanes stride over a window
  // of xH * xKBH ring entries; the label rows of its ring are xRLP >= K +
  // xH * xKBH entries apart, padded so that a half warp's 64-bit reads of
  // consecutive entries of different labels fall in distinct banks.
  int xRLP;
  // Posteriors from kept ring values (posterior.cu): cut normaliser every
  // GS positions, ngrid grid points per sequence; the posterior pass stages
  // pRT boundaries (plus K rows of halo) of kept values per tile.
  int GS, ngrid, pRT;
  int pKH;       // segment-end rows staged at once by the posterior pass (K, or a
                 // chunk of the durations for long durations)
  int npch;      // path-score chunks per sequence, ceil(T / PATH_ROWS)
};

// Device pointers into the caller's workspace.
struct WsPtrs {
  int* status;
  int32_t* sint;   // [B][Tstride][C] integer part of the base-2 prefix sums
  float* sfrac;    // [B][Tstride][C] fractional part
  double* chunk;   // [B][nchunk][C] per-chunk emission sums
  double* logz2;   // [B] log2 Z from the forward ring
  double* logz2b;  // [B] log2 Z from the backward ring
  float2* ack;     // [B][nck][K][C] forward ring checkpoints (boundary order)
  double* acf;     // [B][nck] their frame bases
  float2* bck;     // [B][nck][K][C] backward ring checkpoints
  double* bcf;     // [B][nck]
  float* store;    // [B][nck][delta][store_w] recompute store (when not in smem)
  double* pgt;     // [B][nck][C][C] transition-count partials
  double* pgd;     // [B][nck][K][C] duration-count partials
  double* segT;    // [B][nck][C] per-segment sum of (start - end) marginals
  double* segV;    // [B][nck][C] per-segment sum of the within-segment suffix sums
  int32_t* bp;     // [B][T+1][C] Viterbi backpointers (viterbi_pipe: the chosen duration only)
  float* vrow;     // [B][T+1][C] viterbi_pipe: V per boundary, relative to its frame
  int32_t* wrd;    // [B][T+1][CP] viterbi_pipe: backpointer words, CP = C rounded up to 4
  int32_t* varg;   // [B][T+1][CP] viterbi_pipe: label argmax A[s, c] of a segment starting at s
  float* kv;       // [B][2][T+1][2][C] exponential-domain ring values per boundary:
                   //   direction (forward, backward) x (p, acc), relative to the frame
  double* kf;      // [B][2][T+1] that frame (absolute, log2 units)
  double* ncut;    // [B][ngrid] log2 of the cut normaliser at the grid positions
  float* emax;     // [B] largest |centred emission| * log2(e) over the valid positions
  int* mode;       // [2][B] ring path per (direction, sequence): 1 exponential, 2 log domain
  float* tmax;     // [1] M = max trans * log2(e), written by the exponential-domain rings
  // Path score (path.cu); a region of its own, so that it may run between a
  // forward and its backward on the same workspace.
  // pcnt, pbad and pdone are one contiguous region, zeroed by one memset
  // before every call (pzero_bytes).
  int32_t* pcnt;   // [B][C*C + K*C] gold transition then duration counts
  double* psum;    // [B][npch][C] per-chunk emission column sums
  int32_t* plab;   // [B][npch][C] per-chunk label counts
  double* pscr;    // [B][npch] per-chunk sum of the gold terms
  double* pfr;     // [B][C] n_c / L_b (0 without centering)
  double* pw;      // [B] gradient weight (0 for a malformed path)
  int32_t* pbad;   // [B] malformed-path bits
  int32_t* pdone;  // [B] chunks of the sequence finished (the last one reduces)
  // Boundary projections: pd[b][t][c] = P_end[t-1, c] + P_start[t, c] in
  // base-2 units (the start side of boundary t; the end side P_end[t-1] is
  // folded into the stored prefix sums), read when *pon != 0 (pon is the
  // word after the status word, cleared with it by every forward / decode).
  int* pon;
  float* pd;       // [B][Tstride][C]
  size_t pzero_bytes;
};

}  // namespace semicrf
