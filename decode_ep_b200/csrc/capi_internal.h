// Internal helpers shared by the C-ABI translation units of libentropack.
#pragma once

#include <cstdint>

#include <cuda_runtime.h>

#include "entropack.h"

namespace epk {

// Records the calling thread's last error message (printf-style) and returns st.
ep_status fail(ep_status st, const char* fmt, ...);

// Clears the calling thread's last error message.
void clear_error();

// CRC-32 (IEEE 802.3, reflected polynomial 0xEDB88320), table-driven.
uint32_t crc32(const uint8_t* p, uint64_t n);

// Full host validation of a blob (header, sections, tables, offsets, CRC).
ep_status validate_blob(const uint8_t* blob, uint64_t bytes);

// The library's stream-ordered scratch pool on the current device, created on first use. Freed
// scratch up to 1 GiB stays mapped for the next call; above that it goes back at the next
// synchronisation.
cudaError_t scratch_pool(cudaMemPool_t* out);

}  // namespace epk
