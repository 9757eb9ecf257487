// m3_scan_plan.cuh -- the segment plan shared by the chunked scan kernels.
//
// With fewer (batch, head) sequences than CTA slots a sequence is cut into nseg segments of
// seg_tiles tiles.  A state pass summarises segments 0..nseg-2, cut into nsub sub-segments in
// all, each from a zero start: its end state, total log decay and total rotation angle.  The
// full pass starts segment k from the sequence's incoming state folded through the summaries
// of the sub-segments before it.  The workspace holds the incoming state (ws_init) and the
// summaries.
#pragma once

#include <stdint.h>

namespace m3 {

struct SegInfo {
  int nseg;        // full-pass segments per sequence
  int seg_tiles;   // tiles per full-pass segment
  int nsub;        // state-pass sub-segments per sequence: they tile segments 0..nseg-2
  int sub_tiles;   // tiles per sub-segment (divides seg_tiles)
  float* ws_init;  // (b*H, N, P): rotated-frame state entering segment 0 (nseg > 1)
  float* ws_h;     // (b*H, nsub, N, P): end state of each sub-segment from a zero start
  float* ws_l;     // (b*H, nsub): total log decay of each sub-segment
  double* ws_phi;  // (b*H, nsub, N/2): total angle of each sub-segment, reduced mod 2 pi
  int write_init;  // state pass: sub-segment 0 writes the state's h+ to ws_init (0: a range
                   // summary, which reads no incoming state)
};

// The MIMO rank a chunked tensor-core kernel runs a rank R at: the next of 1, 2, 4, 8.  Branches
// R .. rank-1 are zero padding: their B and C rows are the zero fill of the tile copies and their
// W_x, W_o and biases are zero, so they add nothing to the state or the output.
__host__ __device__ inline int tile_rank(int R) { return R <= 1 ? 1 : R <= 2 ? 2 : R <= 4 ? 4 : 8; }

}  // namespace m3
