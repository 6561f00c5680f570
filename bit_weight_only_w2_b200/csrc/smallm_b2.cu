// Instantiations of the small-M kernel for 2-bit codes (both group sizes, 1..16 octets per tile).
#include <utility>

#include "smallm_kernel.cuh"

LOWBIT_SMALLM_TABLE(2)
