// Host-side interface of the fused single-token decode stack, shared by the
// stack object (stack.cu) and the kernel's translation unit (stack_decode.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "qmoe.h"

namespace qmoe {

struct FusedPlan {
  size_t smem;
  int nslots, slot_bytes;
  int ncons;   // consumer warps that take ring items (nslots is a multiple of it)
};

// Device buffers of the fused path, carved from the stack's workspace.
struct FusedBufs {
  float *wrt;                      // [L][H][E] transposed routers
  unsigned long long *lacc;         // [2][E] integer partial-logit sums (2^-32 units)
  double *ssq;                     // [copies][2][H/16] slice sums of squares
  float *zbuf;                     // [copies][2][H] residual stream z
  uint8_t *lbuf;                   // limbs of h, [k][I/32][96]
  float2 *lscg;                    // block scales of h, [k][I/32]
  unsigned *bar;
  const uint8_t **gu, **dn;
  const float **bias;
  int32_t *fmt;                    // [L] block format of each layer
};

// fmt: the stack's one block format, or QMOE_Q4 for a stack that mixes
// formats (its shared-memory layout is the widest format's).
bool fused_stack_plan(int fmt, int E, int H, int I, int k, FusedPlan *p);
size_t fused_stack_ws_bytes(int L, int E, int H, int I, int k);
FusedBufs fused_carve(void *ws, int L, int E, int H, int I, int k);
qmoe_status fused_prepare(const FusedBufs &b, int L, int E, int H, const float *const *Wr,
                          const qmoe_experts *layers, const float *const *bias, cudaStream_t s);
// fmt: the stack's block format, or 0 when the layers mix formats (the kernel
// then reads each layer's format from the prepared table).
// trace: null, or [L][grid][fused_trace_points()] int64 SM-clock stamps per
// layer and CTA (layer start, top-k done, gate/up tiles start and done, first
// grid barrier passed, down tiles done, second grid barrier passed).
qmoe_status fused_launch(const FusedBufs &b, const FusedPlan &p, int fmt, int L, int E, int H, int I, int k, float eps,
                         const float *x_in, float *x_out, int32_t *idx_rec, float *gate_rec, int32_t *status,
                         long long *trace, cudaStream_t s, bool cooperative);
int fused_trace_points();

}  // namespace qmoe
