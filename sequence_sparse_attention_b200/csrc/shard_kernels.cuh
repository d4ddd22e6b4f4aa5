// shard_kernels.cuh -- data movement of the sharded layer (one ZigZag physical
// host per GPU): the batched 2-D copies that pack a rank's passing blocks and
// query-row partials into its exchange messages and unpack every rank's
// messages after the all-gathers.
//
// "Riepilogo Tecnico: APB-V", Ottimizzazioni a Livello di Sistema,
// "Comunicazione Sovrapposta": each host's passing blocks travel to the hosts
// after it, and "Forward Fuso di Contesto e Query": the query rows' partial
// results of every host are merged through their log-sum-exp.  The collective
// itself runs between the library's calls (the caller's NCCL all-gather into
// this GPU's own memory); these kernels only move bytes within one GPU.
#pragma once

#include <stdint.h>

namespace spava {

// One 2-D copy: `height` rows of `width` bytes, row r from src + r*src_pitch
// to dst + r*dst_pitch.  unit = 16 (every address, pitch and width a multiple
// of 16) or 4 (multiples of 4).
struct CopyJob {
    const char *src;
    char *dst;
    int64_t src_pitch, dst_pitch;
    int32_t width, height, unit, pad;
};
constexpr int kMaxCopyJobs = 64;
struct CopyBatch {
    CopyJob job[kMaxCopyJobs];
    int32_t n;
};

// blockIdx.y = job; the job's units (width/unit per row x height rows) are
// spread over gridDim.x blocks with a grid-stride loop.
__global__ void __launch_bounds__(256) batched_copy_kernel(const __grid_constant__ CopyBatch B) {
    const CopyJob &j = B.job[blockIdx.y];
    const int64_t per_row = j.width / j.unit;
    const int64_t total = per_row * j.height;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < total; i += stride) {
        const int64_t r = i / per_row, c = i - r * per_row;
        if (j.unit == 16) {
            const uint4 x = *reinterpret_cast<const uint4 *>(j.src + r * j.src_pitch + c * 16);
            *reinterpret_cast<uint4 *>(j.dst + r * j.dst_pitch + c * 16) = x;
        } else {
            const uint32_t x = *reinterpret_cast<const uint32_t *>(j.src + r * j.src_pitch + c * 4);
            *reinterpret_cast<uint32_t *>(j.dst + r * j.dst_pitch + c * 4) = x;
        }
    }
}

}  // namespace spava
