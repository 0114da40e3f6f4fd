/* Plain-C consumer of include/bitlinear.h: compiled with a C compiler and
 * linked against libbitlinear.so by tests/test_c_abi.py.  It calls only
 * entry points that answer without a GPU: the version, the status strings,
 * the size queries, and calls whose arguments are rejected on the host. */
#include <stdio.h>
#include <string.h>

#include "bitlinear.h"

int main(void) {
  int bad = 0;
  if (bl_version() < 100) bad |= 1;
  if (strcmp(bl_status_string((bl_status)99), "unknown status") != 0) bad |= 2;
  if (bl_packed_weight_bytes(6912, 2560) != (size_t)6912 * 2560 / 4) bad |= 4;
  if (bl_forward_workspace_bytes(4096, 2560, 6912, 8) < (size_t)4096 * 2560) bad |= 8;
  if (bl_forward_rmsnorm_workspace_bytes(1, 2560, 6912, 8) < 2560) bad |= 16;
  /* K not a multiple of 64: rejected before any CUDA call */
  if (bl_forward((const uint16_t*)0x10000, 1, 100, 8, (const uint8_t*)0x10000, (const float*)0x10000, 8,
                 (uint16_t*)0x10000, NULL, 0, (cudaStream_t)0) != BL_ERR_SHAPE)
    bad |= 32;
  /* eps must be positive */
  if (bl_forward_rmsnorm((const uint16_t*)0x10000, NULL, 0.0f, 1, 64, 8, (const uint8_t*)0x10000,
                         (const float*)0x10000, 8, (uint16_t*)0x10000, (void*)0x10000, 1 << 20,
                         (cudaStream_t)0) != BL_ERR_INVALID_ARG)
    bad |= 64;
  /* LayerNorm: eps must be positive; the grouped form takes no weights */
  if (bl_forward_layernorm((const uint16_t*)0x10000, -1.0f, 1, 64, 8, (const uint8_t*)0x10000, (const float*)0x10000,
                           8, (uint16_t*)0x10000, (void*)0x10000, 1 << 20, (cudaStream_t)0) != BL_ERR_INVALID_ARG)
    bad |= 128;
  {
    bl_linear p = {(const uint16_t*)0x10000, 1, 64, 8, (const uint8_t*)0x10000, (const float*)0x10000,
                   (uint16_t*)0x10000};
    const uint16_t* w[1] = {(const uint16_t*)0x10000};
    if (bl_forward_norm_grouped(1, &p, BL_NORM_LAYER, w, 1e-5f, 8, (void*)0x10000, 1 << 20, (cudaStream_t)0) !=
        BL_ERR_INVALID_ARG)
      bad |= 256;
  }
  printf("c abi check: %s (%d)\n", bad ? "FAILED" : "ok", bad);
  return bad ? 1 : 0;
}
