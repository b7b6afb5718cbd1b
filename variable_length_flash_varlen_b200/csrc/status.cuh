// Device status word shared by every kernel of the library (one translation
// unit): bounded waits that give up and schedule overflows OR their bit in.
#pragma once

namespace va {
__device__ unsigned g_va_status = 0;
}  // namespace va
