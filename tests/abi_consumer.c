/*
 * abi_consumer.c -- a plain C99 user of libvggt_attn.so: include/vggt_attn.h
 * compiled as C (no C++ anywhere), every declared entry point resolved at link
 * time, and the host-side rules of the header exercised without a GPU (every
 * call below either needs no device or fails its argument checks before
 * touching one). Built and run by tests/test_abi_c.py; prints "ok" and
 * returns 0, or names the first failed check and returns 1.
 */
#include <stdio.h>
#include <string.h>

#include "vggt_attn.h"

static int failures = 0;

#define CHECK(cond)                                                    \
    do {                                                               \
        if (!(cond)) {                                                 \
            fprintf(stderr, "check failed, line %d: %s\n", __LINE__, #cond); \
            ++failures;                                                \
        }                                                              \
    } while (0)

/* Every entry point of the header, taken by address: the program links only if
   the library exports each of them with C linkage. */
typedef void (*vggt_fn)(void);
static const vggt_fn entry_points[] = {
    (vggt_fn)&vggt_attn_frame,         (vggt_fn)&vggt_attn_global,
    (vggt_fn)&vggt_attn_descriptor,    (vggt_fn)&vggt_qk_prologue,
    (vggt_fn)&vggt_attn_core,          (vggt_fn)&vggt_attn_core_online,
    (vggt_fn)&vggt_kv_pool,            (vggt_fn)&vggt_desc_cache_create,
    (vggt_fn)&vggt_desc_cache_destroy, (vggt_fn)&vggt_desc_cache_frames,
    (vggt_fn)&vggt_desc_cache_reset,   (vggt_fn)&vggt_attn_descriptor_chunk,
    (vggt_fn)&vggt_attn_frame_ex,      (vggt_fn)&vggt_attn_global_ex,
    (vggt_fn)&vggt_attn_descriptor_ex, (vggt_fn)&vggt_attn_subset,
    (vggt_fn)&vggt_attn_frame_f32,     (vggt_fn)&vggt_attn_global_f32,
    (vggt_fn)&vggt_attn_global_batch,  (vggt_fn)&vggt_attn_descriptor_batch,
    (vggt_fn)&vggt_kv_pool_ex,         (vggt_fn)&vggt_kv_pool_tokens_ex,
    (vggt_fn)&vggt_qk_prologue_ex,     (vggt_fn)&vggt_descriptor_keys,
    (vggt_fn)&vggt_desc_cache_create_ex, (vggt_fn)&vggt_attn_global_noalloc,
    (vggt_fn)&vggt_kv_pool_tokens,     (vggt_fn)&vggt_get_device_status,
    (vggt_fn)&vggt_release_scratch,    (vggt_fn)&vggt_scratch_pool_info,
    (vggt_fn)&vggt_status_string,      (vggt_fn)&vggt_set_wait_limit,
    (vggt_fn)&vggt_debug_wait_timeout,
};

int main(void) {
    /* a 16-byte aligned address that is never dereferenced: every call that
       receives it fails validation first */
    vggt_bf16* const fake = (vggt_bf16*)(uintptr_t)0x1000;
    float* const fake_pos = (float*)(uintptr_t)0x2000;
    size_t i;

    for (i = 0; i < sizeof entry_points / sizeof entry_points[0]; ++i) CHECK(entry_points[i] != NULL);

    /* status strings */
    CHECK(strncmp(vggt_status_string(VGGT_OK), "VGGT_", 5) == 0);
    CHECK(strncmp(vggt_status_string(VGGT_ERR_RANGE), "VGGT_", 5) == 0);

    /* pooled token counts: 5 specials + ceil(g / kv_down)^2 cells */
    CHECK(vggt_kv_pool_tokens(1374, 4) == 105);
    CHECK(vggt_kv_pool_tokens(4101, 4) == VGGT_N_SPECIAL + 16 * 16);
    CHECK(vggt_kv_pool_tokens(930, 4) == VGGT_ERR_SHAPE); /* 25 x 37 is not square */
    {
        vggt_frame_layout L;
        memset(&L, 0, sizeof L);
        L.n_front = 5;
        L.grid_h = 25;
        L.grid_w = 37;
        L.n_back = 0;
        CHECK(vggt_kv_pool_tokens_ex(930, 4, &L) == 5 + 7 * 10);
    }

    /* argument checks, before any device access */
    CHECK(vggt_attn_global(NULL, fake, fake, fake_pos, fake, 2, 261, 16, 64, 1, 0) == VGGT_ERR_NULL);
    CHECK(vggt_attn_global(fake, fake, fake, fake_pos, fake, 2, 261, 16, 32, 1, 0) == VGGT_ERR_UNSUPPORTED);
    CHECK(vggt_attn_frame(fake, fake, fake, fake_pos, fake, 2, 262, 16, 64, 1, 0) == VGGT_ERR_SHAPE);
    CHECK(vggt_attn_descriptor(fake, fake, fake, fake_pos, fake, 2, 261, 16, 64, 0, 0) == VGGT_ERR_SHAPE);
    CHECK(vggt_attn_global(fake + 4, fake, fake, fake_pos, fake, 2, 261, 16, 64, 1, 0) ==
          VGGT_ERR_UNSUPPORTED); /* 8-byte offset: not 16-byte aligned */
    CHECK(vggt_attn_global(fake, fake, fake, fake_pos, fake, 1 << 20, 261, 16, 64, 1, 0) == VGGT_ERR_SHAPE);
    CHECK(vggt_kv_pool(fake, fake, fake_pos, fake, fake, fake_pos, 2, 261, 16, 64, 0, 0) == VGGT_ERR_SHAPE);
    CHECK(vggt_qk_prologue(fake, NULL, fake, 10, 16, 64, 0) == VGGT_ERR_NULL);

    /* empty problems succeed without touching a pointer */
    CHECK(vggt_attn_global(NULL, NULL, NULL, NULL, NULL, 0, 261, 16, 64, 1, 0) == VGGT_OK);
    CHECK(vggt_kv_pool(NULL, NULL, NULL, NULL, NULL, NULL, 0, 261, 16, 64, 4, 0) == VGGT_OK);

    if (failures) return 1;
    printf("ok\n");
    return 0;
}
