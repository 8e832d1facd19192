/* The C ABI used from plain C (no Python, no device): problem validation and
 * workspace sizing, status strings, and the selector-artifact reader on a
 * file this program writes.  Exit status 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "veda.h"

#define CHECK(cond)                                                        \
    do {                                                                   \
        if (!(cond)) {                                                     \
            fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
            return 1;                                                      \
        }                                                                  \
    } while (0)

static veda_problem problem(void)
{
    veda_problem p;
    memset(&p, 0, sizeof p);
    p.B = 1; p.H = 2; p.d = 128; p.tile = 128; p.r = 64;
    p.dtype = VEDA_BF16;
    p.q = (const void*)(uintptr_t)0x100000;
    const int64_t n = 1000;
    p.q_stride_b = n * 2 * 128; p.q_stride_tok = 2 * 128; p.q_stride_h = 128;
    p.video.k = (const void*)(uintptr_t)0x200000;
    p.video.v = (const void*)(uintptr_t)0x300000;
    p.video.n_tokens = n;
    p.video.stride_b = n * 2 * 128; p.video.stride_tok = 2 * 128; p.video.stride_h = 128;
    p.video.budget = 2;
    return p;
}

int main(int argc, char** argv)
{
    if (argc < 2) return 2;
    size_t bytes = 0;
    veda_problem p = problem();
    CHECK(veda_workspace_size(&p, &bytes) == VEDA_OK && bytes > 256);
    p.d = 96;
    CHECK(veda_workspace_size(&p, &bytes) == VEDA_ERR_UNSUPPORTED);
    p = problem();
    p.video.budget = 9;   /* 1000 tokens = 8 tiles */
    CHECK(veda_workspace_size(&p, &bytes) == VEDA_ERR_INVALID_ARG);
    CHECK(strcmp(veda_status_string(VEDA_ERR_FORMAT), "VEDA_ERR_FORMAT") == 0);

    /* a one-tensor safetensors file: F16 [2, 3] */
    const char* path = argv[1];
    const char header[] = "{\"w\":{\"dtype\":\"F16\",\"shape\":[2,3],\"data_offsets\":[0,12]},"
                          "\"__metadata__\":{\"hotkey\":\"abc\"}}";
    const uint64_t hlen = sizeof header - 1;
    const uint16_t data[6] = {0x3C00, 0x4000, 0xC200, 0x0000, 0x3800, 0x7C00};  /* 1 2 -3 0 0.5 inf */
    FILE* f = fopen(path, "wb");
    CHECK(f != NULL);
    for (int i = 0; i < 8; ++i) fputc((int)((hlen >> (8 * i)) & 0xFF), f);
    fwrite(header, 1, hlen, f);
    fwrite(data, sizeof data, 1, f);
    fclose(f);

    veda_selector* s = NULL;
    CHECK(veda_selector_open(path, &s) == VEDA_OK);
    CHECK(veda_selector_count(s) == 1);
    const int64_t shape[2] = {2, 3};
    CHECK(veda_selector_check(s, 1, shape, 2, 1000, "hotkey") == VEDA_OK);
    CHECK(veda_selector_check(s, 100, shape, 2, 0, NULL) == VEDA_ERR_FORMAT);
    CHECK(strcmp(veda_selector_metadata(s, "hotkey"), "abc") == 0);
    float out[6];
    CHECK(veda_selector_read(s, 0, VEDA_F32, 1.0f, out, sizeof out) == VEDA_OK);
    CHECK(out[0] == 1.0f && out[1] == 2.0f && out[2] == -3.0f && out[3] == 0.0f && out[4] == 0.5f);
    CHECK(out[5] > 3.0e38f);
    veda_selector_close(s);
    CHECK(veda_selector_open("/nonexistent/selector.safetensors", &s) == VEDA_ERR_IO);
    printf("ok\n");
    return 0;
}
