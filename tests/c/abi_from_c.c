/* The C ABI used from plain C (no CUDA headers, no torch): every call here is
 * host-only or rejected before a launch, so it runs on a machine without a GPU.
 * Compiled with -Werror against include/lightning.h, so the header's
 * declarations must be valid C and must match the exported symbols at link
 * time. Exit status 0 and "ok" when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "lightning.h"

static int failures = 0;

static void check(int cond, const char *what) {
    if (!cond) {
        fprintf(stderr, "FAILED: %s (last error: %s)\n", what, lightning_last_error_message());
        ++failures;
    }
}

/* fake, 16-byte aligned, non-overlapping device addresses: never dereferenced */
static const void *fake(int i) { return (const void *)(uintptr_t)(0x10000000u * (unsigned)(i + 1)); }

int main(void) {
    check(lightning_abi_version() == 2, "ABI version 2");
    for (int s = LA_OK; s <= LA_ERR_TIMEOUT; ++s)
        check(lightning_status_string(s) != NULL && strlen(lightning_status_string(s)) > 0, "status strings");

    check(lightning_prefill_snapshot_count(131072, 16384) == 8, "snapshot count");
    check(lightning_prefill_snapshot_count(-1, 16) == -1, "snapshot count of a bad length");
    check(lightning_prefill_workspace_size(1, 64, 131072, 128, 256) == 64 * 48,
          "the CTA-pair prefill's workspace: 48 bytes per (batch, head)");
    check(lightning_prefill_workspace_size(1, 64, 131072, 128, 128) == 64 * 48,
          "the single-CTA prefill's workspace: 48 bytes per (batch, head)");
    check(lightning_prefill_backward_noalloc_capacity() > 0, "no-alloc backward capacity");
    check(lightning_gqa_decode_workspace_size(8, 64, 131072) > 0, "GQA decode workspace");
    check(lightning_prefill_selected_variant(LA_DTYPE_BF16, 1, 64, 131072, 128, 256, LA_VARIANT_AUTO) ==
              LA_VARIANT_TCGEN05_PAIR, "bf16 / d128 / B256 runs on the CTA pair");
    check(lightning_prefill_selected_variant(LA_DTYPE_F32, 1, 2, 256, 64, 64, LA_VARIANT_AUTO) == LA_VARIANT_SIMT,
          "float32 runs on CUDA cores");

    float *state = (float *)fake(5), *state_out = (float *)fake(6);
    const float *slopes = (const float *)fake(4);
    void *o = (void *)fake(3);
    /* rejected before any launch */
    check(lightning_prefill(fake(0), fake(1), fake(2), LA_DTYPE_BF16, slopes, 1, 2, 16, 96, 256, NULL, o, state_out,
                            NULL, 0, NULL) == LA_ERR_UNSUPPORTED, "dim 96 unsupported");
    check(lightning_prefill(fake(0), fake(1), fake(2), LA_DTYPE_BF16, slopes, 1, 2, 16, 128, 256, NULL, (void *)fake(0),
                            state_out, NULL, 0, NULL) == LA_ERR_INVALID_ARG, "o overlapping q");
    check(lightning_prefill(fake(0), fake(1), fake(2), LA_DTYPE_BF16, slopes, 1, 2, 16, 128, 256, NULL, o, state_out,
                            NULL, 0, NULL) == LA_ERR_INVALID_ARG, "the CTA-pair prefill without its workspace");
    check(lightning_prefill(fake(0), fake(1), fake(2), LA_DTYPE_BF16, slopes, 1, 2, 16, 128, 128, NULL, o, state_out,
                            NULL, 0, NULL) == LA_ERR_INVALID_ARG, "the single-CTA prefill without its workspace");
    check(lightning_decode(fake(0), fake(1), fake(2), (la_dtype)7, slopes, 1, 2, 128, state, o, NULL) ==
              LA_ERR_INVALID_ARG, "bad dtype");
    check(lightning_prefill_norm_gate(fake(0), fake(1), fake(2), LA_DTYPE_F32, slopes, 1, 2, 16, 128, 256, NULL,
                                      fake(7), (const float *)fake(8), 1e-6f, (void *)fake(9), NULL, NULL, 0,
                                      NULL) ==
              LA_ERR_UNSUPPORTED, "fused norm + gate needs bf16");
    /* nothing to do: returns before touching the device */
    check(lightning_prefill(fake(0), fake(1), fake(2), LA_DTYPE_BF16, slopes, 0, 2, 16, 128, 256, NULL, o, state_out,
                            NULL, 0, NULL) == LA_OK, "empty batch");

    if (failures) return 1;
    printf("ok\n");
    return 0;
}
