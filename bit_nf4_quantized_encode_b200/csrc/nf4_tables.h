// nf4_tables.h -- host-side tables of the CUDA library: the NF4 codebook, the
// decision thresholds between neighbouring levels, and the bucketed lookup
// table the encode kernel uses to pick a code with one comparison.
#pragma once
#include <cstdint>

namespace qlora {

// Buckets of the normalized value n in [-1, 1]: u = RN(16 n + 16) in [0, 32].
constexpr int kNumBuckets = 33;

struct Nf4Tables {
  float level[16];            // levels, ascending (FP4 repeats +1 in the last entry)
  float threshold[15];        // code(n) = #{i : n >= threshold[i]}
  float bucket_thr[kNumBuckets];     // the one threshold inside bucket u, or +inf
  uint8_t bucket_base[kNumBuckets];  // code of the smallest n in bucket u
  // Fast-path word of bucket u: the threshold's float bits with the low five
  // mantissa bits replaced by bucket_base[u] + 1 (a bucket without a threshold
  // gets a huge finite float); the perturbation is below 2^-19.
  uint32_t bucket_fast[kNumBuckets];
  bool ok;                    // every bucket holds at most one threshold
  bool fast_ok;               // every threshold lies more than 2^-18 inside its bucket
};

// The 4-bit data types: the values of qlora_nf4_tensor::quant_type.
constexpr int kTypeNf4 = 0;
constexpr int kTypeFp4 = 1;
constexpr int kTypeInt4 = 2;
constexpr int kNumTypes = 3;

// The tables of one type (NF4 for an unknown type), all built once
// (thread-safe) on first use.
const Nf4Tables& level_tables(int type);
const Nf4Tables& nf4_tables();

}  // namespace qlora
