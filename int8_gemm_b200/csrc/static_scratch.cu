// Built-in scratch memory of bs_int_scaled_mm_noalloc: the stream-K
// partial-sum slots and flag words of the wide kernel in a fixed array of this
// module, laid out as a registered workspace is (slots of kWsSlotWords words,
// one per CTA, then the flag words), for devices of up to
// kStaticScratchMaxSms SMs.
//
// It sits in a translation unit of its own, so its module (and the 20 MB of
// device memory the array takes) is loaded only by a process that asks for
// the array's address.
#include "launch.h"

namespace bsg {

static __device__ __align__(256) uint8_t g_split_scratch[kStaticScratchBytes];

cudaError_t static_scratch_address(void** ptr) { return cudaGetSymbolAddress(ptr, g_split_scratch); }

}  // namespace bsg
