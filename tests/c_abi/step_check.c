/* A plain C program that runs the fused step through the C ABI with device
 * memory from the CUDA runtime (no Python, no torch), and checks the first
 * step against its closed form: at t = 1 the bias corrections give
 * m_hat = g and v_hat = g^2, so AdamW moves w by -lr * (g / (|g| + eps) +
 * lambda * w) for any reduced gradient g ("Deep dive: DeepSpeed", the scalar
 * Adam of "Reduce first, then update the owned slice"; decoupled decay of the
 * "ZeRO" page's AdamW).  Exit status 0 when every element holds. */
#include <math.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "zero_adam.h"

#define NPARAM 100003
#define NRANK 4
#define GSTRIDE 100008 /* NPARAM rounded up to 8: every rank's gradient starts 16-byte aligned */

static int cuda_ok(cudaError_t e, const char* what) {
    if (e != cudaSuccess) fprintf(stderr, "%s: %s\n", what, cudaGetErrorString(e));
    return e == cudaSuccess;
}

static uint16_t bf16_rne(float x) {  /* round-to-nearest-even of a finite float to bfloat16 */
    uint32_t b;
    memcpy(&b, &x, 4);
    b += 0x7FFFu + ((b >> 16) & 1u);
    return (uint16_t)(b >> 16);
}

int main(void) {
    const double lr = 1e-3, b1 = 0.9, b2 = 0.999, eps = 1e-8, wd = 0.01;
    float *hg = malloc(sizeof(float) * GSTRIDE * NRANK), *hw = malloc(sizeof(float) * NPARAM);
    float *ow = malloc(sizeof(float) * NPARAM), *om = malloc(sizeof(float) * NPARAM), *ov = malloc(sizeof(float) * NPARAM);
    uint16_t* op = malloc(sizeof(uint16_t) * NPARAM);
    if (!hg || !hw || !ow || !om || !ov || !op) return 2;
    for (int i = 0; i < NPARAM; ++i) {
        hw[i] = (float)(0.02 * sin(0.37 * i));
        for (int r = 0; r < NRANK; ++r) hg[r * GSTRIDE + i] = (float)(((i * 7 + r * 13) % 101 - 50) * 1e-4);
    }
    void *grads_dev = NULL, *w = NULL, *m = NULL, *v = NULL, *p16 = NULL, *ctrl = NULL, *ws = NULL;
    if (!cuda_ok(cudaMalloc(&grads_dev, sizeof(float) * GSTRIDE * NRANK), "cudaMalloc") ||
        !cuda_ok(cudaMalloc(&w, sizeof(float) * NPARAM), "cudaMalloc") ||
        !cuda_ok(cudaMalloc(&m, sizeof(float) * NPARAM), "cudaMalloc") ||
        !cuda_ok(cudaMalloc(&v, sizeof(float) * NPARAM), "cudaMalloc") ||
        !cuda_ok(cudaMalloc(&p16, sizeof(uint16_t) * NPARAM), "cudaMalloc") ||
        !cuda_ok(cudaMalloc(&ctrl, zero_ctrl_bytes()), "cudaMalloc") ||
        !cuda_ok(cudaMalloc(&ws, zero_workspace_bytes()), "cudaMalloc"))
        return 2;
    cudaMemcpy(grads_dev, hg, sizeof(float) * GSTRIDE * NRANK, cudaMemcpyHostToDevice);
    cudaMemcpy(w, hw, sizeof(float) * NPARAM, cudaMemcpyHostToDevice);
    cudaMemset(m, 0, sizeof(float) * NPARAM);
    cudaMemset(v, 0, sizeof(float) * NPARAM);
    if (zero_ctrl_init(ctrl, 1.0f, NULL) || zero_workspace_init(ws, NULL) ||
        zero_gather_params(w, p16, ZERO_BF16, NPARAM, NULL)) {
        fprintf(stderr, "init failed: %s\n", zero_last_cuda_error());
        return 2;
    }
    const void* grads[NRANK];
    for (int r = 0; r < NRANK; ++r) grads[r] = (const char*)grads_dev + sizeof(float) * (size_t)GSTRIDE * r;
    zero_step_args a;
    memset(&a, 0, sizeof a);
    a.P = NPARAM;
    a.R = NRANK;
    a.owner = -1;
    a.grad_dtype = ZERO_F32;
    a.param_dtype = ZERO_BF16;
    a.grads = grads;
    a.master[0] = w;
    a.exp_avg[0] = m;
    a.exp_avg_sq[0] = v;
    a.params16 = p16;
    a.hp.lr = lr;
    a.hp.beta1 = b1;
    a.hp.beta2 = b2;
    a.hp.eps = eps;
    a.hp.weight_decay = wd;
    a.ctrl = ctrl;
    a.workspace = ws;
    int rc = zero_step_fused(&a, NULL);
    if (rc != ZERO_OK || !cuda_ok(cudaDeviceSynchronize(), "step")) {
        fprintf(stderr, "zero_step_fused: %s (%s)\n", zero_status_string(rc), zero_last_cuda_error());
        return 2;
    }
    cudaMemcpy(ow, w, sizeof(float) * NPARAM, cudaMemcpyDeviceToHost);
    cudaMemcpy(om, m, sizeof(float) * NPARAM, cudaMemcpyDeviceToHost);
    cudaMemcpy(ov, v, sizeof(float) * NPARAM, cudaMemcpyDeviceToHost);
    cudaMemcpy(op, p16, sizeof(uint16_t) * NPARAM, cudaMemcpyDeviceToHost);
    zero_ctrl c;
    zero_ctrl_read(ctrl, &c, NULL);
    int bad = 0;
    for (int i = 0; i < NPARAM; ++i) {
        double g = 0.0;
        for (int r = 0; r < NRANK; ++r) g += (double)hg[r * GSTRIDE + i];
        g /= NRANK;
        const double w0 = hw[i];
        const double w1 = w0 - lr * (g / (fabs(g) + eps) + wd * w0);
        const double m1 = (1.0 - b1) * g, v1 = (1.0 - b2) * g * g;
        if (fabs(ow[i] - w1) > 1e-5 * fabs(w1) + 1e-7 || fabs(om[i] - m1) > 1e-5 * fabs(m1) + 1e-7 ||
            fabs(ov[i] - v1) > 1e-5 * fabs(v1) + 1e-7 || op[i] != bf16_rne(ow[i])) {
            if (bad < 5) fprintf(stderr, "element %d: w %.9g (want %.9g) m %.9g v %.9g\n", i, ow[i], w1, om[i], ov[i]);
            ++bad;
        }
    }
    if (c.step != 1 || c.device_error != 0) ++bad;
    cudaFree(grads_dev);
    cudaFree(w);
    cudaFree(m);
    cudaFree(v);
    cudaFree(p16);
    cudaFree(ctrl);
    cudaFree(ws);
    free(hg);
    free(hw);
    free(ow);
    free(om);
    free(ov);
    free(op);
    if (bad == 0) printf("step_check: first step matches its closed form on %d elements\n", NPARAM);
    return bad == 0 ? 0 : 1;
}
