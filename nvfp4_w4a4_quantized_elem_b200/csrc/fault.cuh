// fault.cuh — the device fault word shared by every kernel of the library.
#pragma once

namespace nvfp4 {

// Nonzero after a bounded wait expired in any kernel; read and cleared by
// nvfp4_read_fault. Bits name the kernel role that gave up.
__device__ unsigned int g_fault_word;

}  // namespace nvfp4
