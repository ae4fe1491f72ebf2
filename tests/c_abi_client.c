/* A plain C99 client of include/bitlinear.h, built and run by
 * tests/test_c_client.py without a GPU: it links libbitlinear.so, calls the
 * host-only entry points and argument checks that return before any device
 * work, and prints what they return (one "name value..." line each). */
#include <stdio.h>

#include "bitlinear.h"

int main(void) {
    int32_t shape[10];
    int i;
    bl_status st;
    printf("version %s\n", bitlinear_version());
    for (i = 0; i <= 5; ++i) printf("status_str %d %s\n", i, bitlinear_status_str((bl_status)i));
    printf("packed_bytes %zu %zu\n", bitlinear_packed_bytes(8640, 3200),
           bitlinear_packed_bytes(3, 5));
    printf("workspace_bytes %zu\n", bitlinear_pack_workspace_bytes());
    printf("packed3_stride %lld %lld\n", (long long)bitlinear_packed3_stride(3200),
           (long long)bitlinear_packed3_stride(1));
    st = bitlinear_decode_shape_for(1, 3200, 8640, 1, 148, shape);
    printf("decode_shape_for %d", (int)st);
    for (i = 0; i < 10; ++i) printf(" %d", (int)shape[i]);
    printf("\n");
    /* argument checks that fail before anything touches a device */
    printf("quant_act_null %d\n",
           (int)bitlinear_quant_act(NULL, BL_BF16, 1, 4, NULL, NULL, NULL, NULL));
    printf("quant_act_empty %d\n",
           (int)bitlinear_quant_act(NULL, BL_BF16, 0, 4, NULL, NULL, NULL, NULL));
    printf("forward_badk %d\n", (int)bitlinear_forward(NULL, NULL, NULL, 1, 0, NULL, NULL, 8,
                                                       NULL, BL_F32, NULL, NULL));
    printf("rmsnorm_f32 %d\n", (int)bitlinear_rmsnorm_quant_act((const void*)256, BL_F32, 1, 4,
                                                                (int8_t*)256, (float*)256,
                                                                (int32_t*)256, NULL));
    return 0;
}
