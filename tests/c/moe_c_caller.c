/* A plain C caller of the library's C ABI (include/moe.h): no Python, no torch.
 * It fills the descriptor of the Mixtral-shaped layer ("Top-k 路由" gate Steps 1-3; Tiny MoE
 * sections 3-8: D = 4096, E = 8 SwiGLU experts of width 14336, softmax top-2 renormalised,
 * dropless) and exercises the host-side entry points that need no GPU: sizing (including the
 * scratch of the small-batch schedule), the Switch capacity rule C = ceil(CF T k / E), and
 * argument validation.  Exit status 0 when every
 * check holds; prints one line per check. */
#include <stdio.h>
#include <string.h>

#include "moe.h"

static int failures = 0;

static void check(int ok, const char* what) {
    printf("%s: %s\n", ok ? "ok" : "FAILED", what);
    if (!ok) ++failures;
}

int main(void) {
    moe_desc_t d;
    memset(&d, 0, sizeof d);
    d.T = 4096; d.D = 4096; d.E = 8; d.F = 14336; d.k = 2;
    d.score = MOE_SCORE_SOFTMAX; d.select = MOE_TOKEN_CHOICE; d.gate = MOE_GATE_RENORM;
    d.overflow = MOE_DROPLESS; d.act = MOE_ACT_SWIGLU; d.dtype = MOE_BF16;
    d.aux_alpha = 0.01f;

    int64_t rows = 0;
    check(moe_rows_max(&d, &rows) == MOE_OK && rows == 4096 * 2, "dropless rows = T * k");
    size_t ws = 0, scratch = 0, bws = 0;
    check(moe_workspace_size(&d, &ws) == MOE_OK && ws > 0, "workspace size");
    check(moe_scratch_size(&d, &scratch) == MOE_OK && scratch > 0 && scratch < ws,
          "step scratch inside the workspace");
    check(moe_backward_workspace_size(&d, &bws) == MOE_OK && bws > 0,
          "backward workspace size");
    printf("workspace %zu B, scratch %zu B, backward workspace %zu B\n", ws, scratch, bws);

    /* Switch-style capacity: ceil(1.25 * 8192 * 1 / 128) = 80 slots per expert */
    moe_desc_t sw = d;
    sw.T = 8192; sw.D = 768; sw.E = 128; sw.F = 3072; sw.k = 1;
    sw.gate = MOE_GATE_RAW; sw.overflow = MOE_CAPACITY_DROP; sw.capacity_factor = 1.25f;
    sw.act = MOE_ACT_RELU;
    int32_t cap = 0;
    check(moe_capacity(&sw, &cap) == MOE_OK && cap == 80, "Switch capacity 80");
    check(moe_rows_max(&sw, &rows) == MOE_OK && rows == 8192, "drop rows = min(T k, E C)");

    /* invalid or unsupported descriptors are refused before anything is launched */
    moe_desc_t bad = d;
    bad.k = 9;
    check(moe_workspace_size(&bad, &ws) == MOE_ERR_INVALID_ARG, "k > E refused");
    bad = d;
    bad.E = 300;
    check(moe_workspace_size(&bad, &ws) == MOE_ERR_UNSUPPORTED, "E > 256 unsupported");
    bad = d;
    bad.n_group = 3; bad.topk_group = 1;
    check(moe_workspace_size(&bad, &ws) == MOE_ERR_INVALID_ARG, "n_group must divide E");
    moe_desc_t f32 = d;
    f32.dtype = MOE_F32;
    check(moe_backward_workspace_size(&f32, &bws) == MOE_OK && bws > 0,
          "fp32 backward workspace size");
    check(moe_layer_forward_train(&f32, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, NULL,
                                  0, NULL) == MOE_ERR_UNSUPPORTED,
          "fp32 training forward refused (the plain forward serves fp32 backward)");
    check(moe_layer_forward(&d, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                            NULL, 0, NULL) != MOE_OK, "null buffers refused");
    check(moe_expert_up_ws(&d, 8, 14336, NULL, 8192, NULL, NULL, NULL, NULL, NULL, 0, NULL) ==
              MOE_ERR_INVALID_ARG, "expert up (scratch form): null buffers refused");
    check(moe_expert_down_ws(&d, 8, 14336, NULL, 8192, NULL, NULL, NULL, NULL, 0, NULL) ==
              MOE_ERR_INVALID_ARG, "expert down (scratch form): null buffers refused");
    /* one token: the scratch also holds the small-batch schedule's k-split partials */
    moe_desc_t one = d;
    one.T = 1;
    size_t sc1 = 0;
    check(moe_scratch_size(&one, &sc1) == MOE_OK && sc1 >= (size_t)8 * 2 * 4096 * 4,
          "one-token scratch holds the down product's partials");
    /* an empty batch: arguments checked, nothing launched, MOE_OK (the pointers below are
     * never dereferenced; the workspace is carved on the host only) */
    moe_desc_t none = d;
    none.T = 0;
    size_t ws0 = 0;
    check(moe_workspace_size(&none, &ws0) == MOE_OK, "empty batch: workspace size");
    const int64_t n0 = moe_kernel_launches();
    void* fake = (void*)(uintptr_t)0x100000;
    check(moe_layer_forward(&none, fake, fake, NULL, fake, fake, fake, NULL, NULL, NULL, fake,
                            fake, ws0, NULL) == MOE_OK && moe_kernel_launches() == n0,
          "empty batch: layer forward returns before any launch");
    check(strlen(moe_status_string(MOE_ERR_TIMEOUT)) > 0, "status strings");
    printf("library %s\n", moe_version());
    return failures == 0 ? 0 : 1;
}
