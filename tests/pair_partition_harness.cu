// Test harness: exposes the CTA-pair kernel's host-side tile partition to the CPU tests.
// It compiles the kernel's own translation unit, so the partition under test is the one
// the library builds; only host code runs (no device, no launch).
#include "twq_pair_sm100.cu"

// bounds must hold pairs + 1 entries; returns nonzero on arguments the kernel's launch
// would never pass (the launch caps the pairs at the run table's size).
extern "C" __attribute__((visibility("default"))) int twq_test_pair_partition(
    int num_items, int col_tiles, int G, int res, int h, int r, int pairs, int* bounds) {
  if (num_items < 0 || col_tiles < 1 || G < 1 || pairs < 1 || pairs > 128 || !bounds) return 1;
  twq::partition_items(num_items, col_tiles, G, res != 0, h != 0, r, pairs, bounds);
  return 0;
}
