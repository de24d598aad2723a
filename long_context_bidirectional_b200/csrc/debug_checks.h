// Bounds predicates of the debug build (-DB2A_DEBUG).  In that build every
// tiled TMA copy and every tcgen05 TMEM access or MMA is checked against
// these before it is issued; a failed check sets a bit in the library's
// device status word and the access is skipped, so a wrong coordinate is
// reported instead of reaching the hardware.  Plain C++ so that the CPU
// tests compile and exercise the same predicates.
#pragma once

#include <stdint.h>

#if defined(__CUDACC__)
#define B2A_HD __host__ __device__
#else
#define B2A_HD
#endif

namespace b2a {

// TMEM columns every kernel of the library allocates (all 512 of the SM).
constexpr int kTmemCols = 512;

// A tiled TMA copy of a box starting at (x, y, z) of a map whose innermost
// extent is nx elements of esz bytes: x must be non-negative, inside the
// extent and 16-byte aligned (x * esz a multiple of 16; an unaligned x is an
// illegal instruction on B200); y and z must lie in [0, ny) and [0, nz),
// where nz is the end of the row range the launch covers (a box may run past
// the tensor's last row, which TMA fills, but must not start outside the
// rows the grid owns).  For 2-D maps pass y = 0, ny = 1.
B2A_HD constexpr bool tma_coords_ok(int x, int esz, int nx, int y, int ny, int z, int nz) {
  return x >= 0 && x < nx && (static_cast<long long>(x) * esz) % 16 == 0 && y >= 0 && y < ny && z >= 0 &&
         z < nz;
}

// The copy's shared-memory destination [dst, dst + bytes) inside the CTA's
// dynamic shared memory [base, base + size), 128-byte aligned (the 128-byte
// swizzle's atom).
B2A_HD constexpr bool smem_box_ok(uint32_t dst, uint32_t bytes, uint32_t base, uint32_t size) {
  return dst >= base && (dst & 127u) == 0 && static_cast<uint64_t>(dst) + bytes <= static_cast<uint64_t>(base) + size;
}

// A warp's tcgen05.ld / tcgen05.st of ``cols`` consecutive 32-bit columns at
// TMEM address ``addr`` (lane << 16 | column): the lane field must be the
// first lane of the warp's quarter (32 * (warp % 4)) and the columns must lie
// inside an allocation of kTmemCols columns starting at column 0.
B2A_HD constexpr bool tmem_ldst_ok(uint32_t addr, int cols, int quarter) {
  return (addr >> 16) == 32u * static_cast<uint32_t>(quarter) && (addr & 0xFFFFu) + static_cast<uint32_t>(cols) <= kTmemCols;
}

// An MMA's TMEM operand (the accumulator D of ``cols`` columns, or A read
// from TMEM): lane field 0, columns inside the allocation.
B2A_HD constexpr bool tmem_operand_ok(uint32_t addr, int cols) {
  return (addr >> 16) == 0u && (addr & 0xFFFFu) + static_cast<uint32_t>(cols) <= kTmemCols;
}

// Accumulator columns of a kind::f16 MMA from its instruction descriptor
// (N is stored as N / 8 in bits 17..22).
B2A_HD constexpr int idesc_n(uint32_t idesc) { return static_cast<int>((idesc >> 17) & 0x3Fu) * 8; }

}  // namespace b2a
