// Plan of a grouped call: many independent Sparse-BitLinear layers (2:4, at most 32
// tokens each) quantised and contracted by one launch each.  The plan is built on the host
// (sbn_group_plan), copied to the device by the caller, and read by the kernels; it holds
// the TMA tensor maps of every layer, the work units of the contraction and the rows of
// the activation quantiser.
#pragma once

#include <cuda.h>
#include <stdint.h>

namespace sbn {

constexpr uint32_t kGroupMagic = 0x474e4253u;  // "SBNG"
constexpr uint32_t kGroupVersion = 1;
constexpr int kGroupMaxTokens = 32;  // tokens per layer in a grouped call
constexpr int kGroupRows = 128;      // weight rows per work unit (one MMA M)
constexpr int kGroupKB = 128;        // logical K per pipeline block

struct GroupHeader {
  uint32_t magic, version;
  int32_t count;   // layers
  int32_t nunits;  // contraction work units
  int32_t ncta;    // CTAs of the contraction launch (one per SM at most)
  int32_t bn;      // accumulator width: 16 or 32 tokens
  int32_t nrows;   // (layer, token) rows of the activation quantiser
  int32_t max_nv;  // largest in / 8 over the layers
  int32_t has_x;   // every layer has a bf16 input X (the grouped quantiser may run)
  int32_t split;   // K parts per row tile (1 = no split)
  int64_t off_probs, off_units, off_cta, off_rows;
  int64_t bytes;      // size of the whole plan
  int64_t ws_bytes;   // workspace the contraction needs (0 without a split)
  int64_t ntickets;   // arrival counters at the start of the workspace
  int64_t ws_part_off;  // byte offset of the partial accumulators in the workspace
  int64_t reserved[3];
};
static_assert(sizeof(GroupHeader) == 128, "plan header is 128 bytes");

// One layer.  The tensor maps cover Xq (box 128 inputs x bn tokens, 128-byte swizzle), the
// codes plane and the meta plane (boxes of 16 bytes x 128 rows).
struct alignas(128) GroupProb {
  CUtensorMap tx, tc, tm;
  const void *X;
  int8_t *Xq;
  float *absmax;
  const float *gamma_eff;
  void *Y;
  int32_t *acc_dbg;
  int64_t T, O, K;
  int64_t ticket_base;  // first arrival counter of this layer's row tiles (split only)
  int64_t part_base;    // first partial tile (int32 units from ws_part_off) (split only)
  int32_t y_is_bf16;
  int32_t nparts;       // K parts per row tile
  int64_t ldx;          // row stride (elements) of X and Xq: K, or more for a K slice
};
static_assert(sizeof(GroupProb) == 512, "plan layer record is 512 bytes");

struct GroupUnit {
  int32_t prob, row_tile, kb0, nkb, part;
  int32_t O, K;  // the layer's shape (so a unit's pipeline needs no other record)
  int32_t pad;
};
static_assert(sizeof(GroupUnit) == 32, "plan unit record is 32 bytes");

struct GroupRow {
  int32_t prob, token;
};

}  // namespace sbn
