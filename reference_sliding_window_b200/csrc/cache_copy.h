// Host/device interface of the cache fill from the packed (teacher-forced)
// layout.  Kept apart from internal.h, which the decode kernel compiles
// from, so that this copy path can change without touching its sources.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace rswa {

// Packed form -> cache: rows [0, Lm[b]) and the last W = min(n, T0) outputs
// (FULL mode: all T0) of sequence b, from K/V laid out [B][seq_stride][H][d].
struct LoadPackedParams {
  void* kc;
  void* vc;
  const void* K;
  const void* V;
  int B, H, S_cap, row_bytes, seq_stride;
  int n, T0, full_mode;
  const int32_t* Lm;   // device [B]
  int32_t* T;          // device step counter (kStepSlots copies), all set to T0
};
cudaError_t launch_load_packed(const LoadPackedParams& p, int max_rows, cudaStream_t stream);

// One chunk of the reference segment: rows [0, rows[b]) of sequence b's chunk
// (K/V laid out [B][H][chunk_stride][d]) go to cache rows
// [Lm[b] - rows[b], Lm[b]) of its slabs, Lm already counting the chunk.
struct LoadChunkParams {
  void* kc;
  void* vc;
  const void* K;
  const void* V;
  int B, H, S_cap, row_bytes, chunk_stride;
  const int32_t* Lm;    // device [B], after the chunk
  const int32_t* rows;  // device [B]
};
cudaError_t launch_load_chunk(const LoadChunkParams& p, int max_rows, cudaStream_t stream);

}  // namespace rswa
