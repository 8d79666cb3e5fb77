// Host-side helpers shared by the forward (bsa_fwd_sm100.cu) and backward
// (bsa_bwd_sm100.cu) translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace bsa {

// TMA map of a [rows, d] bf16 row-major tensor (d a multiple of 64): boxes of 64
// columns x box_rows rows, 128-byte swizzle.  False if the driver entry point or the
// encode fails.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint32_t box_rows, int d = 64);

// Enqueues the kernel that packs a [B, L] uint8 key mask into one 64-bit word per
// (b, key block): bit c set when key 64 j + c is kept.
cudaError_t launch_keybits(const uint8_t* key_mask, unsigned long long* bits, int B, int L, int nb,
                           cudaStream_t s);

// Reads and clears the status word of the backward kernels (current device):
// 0, a negative bsa_status a kernel recorded, or BSA_ERR_CUDA if the read failed.
int bwd_take_status();

// The same for the projection kernels (bsa_proj_sm100.cu).
int proj_take_status();

}  // namespace bsa
