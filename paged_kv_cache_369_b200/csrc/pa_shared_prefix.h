// Key splits of the shared-prefix pass (pa_decode_shared_prefix).
//
// The prefix is attended once for all decoding sequences by the tensor-core
// prefill kernel.  With few query rows per KV head (e.g. MHA, one row per
// sequence) one CTA per KV head would leave most SMs idle, so the prefix's
// 64-key tiles are cut into Z contiguous, non-empty ranges of at least about
// 256 keys; range z is one more grid dimension of the pass and writes its own
// partial (lse, o) into workspace slot z.  The tails use slots Z .. and the
// reduce merges every slot.
#pragma once

namespace pa {

constexpr int kPrefixKeyTile = 64;        // keys per tile of the prefill kernel
constexpr int kPrefixKeysPerSplit = 256;  // at least this many keys per range
constexpr int kMaxPrefixSplits = 8;

// Z for a prefix of prefix_len keys: every range holds
// ceil(tiles / Z) tiles except the last, which is never empty.
inline int prefix_splits(int prefix_len) {
    const int tiles = (prefix_len + kPrefixKeyTile - 1) / kPrefixKeyTile;
    int z = (prefix_len + kPrefixKeysPerSplit - 1) / kPrefixKeysPerSplit;
    if (z > kMaxPrefixSplits) z = kMaxPrefixSplits;
    if (z > tiles) z = tiles;
    if (z < 1) z = 1;
    while (z > 1 && (z - 1) * ((tiles + z - 1) / z) >= tiles) --z;
    return z;
}

}  // namespace pa
