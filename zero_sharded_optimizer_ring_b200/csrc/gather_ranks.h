// The per-layer gather from the ranks' own parameter shards (ZeRO-3 with one GPU per rank).
#pragma once

#include "internal.h"

namespace zero {

// The ranks' fp16 parameter shards: rank k's buffer holds flat elements [kS, (k+1)S).
struct ShardPtrs {
    const uint16_t *rank[kMaxBulkRanks];
};

// dst[j] = element lo + j of the flat buffer whose shard k (S elements) is src.rank[k];
// max_ctas > 0: at most that many persistent CTAs (0: a grid of short blocks)
cudaError_t launch_gather_ranks(const ShardPtrs &src, int64_t S, int64_t lo, int64_t n, uint16_t *dst,
                                int32_t max_ctas, cudaStream_t s);

}  // namespace zero
