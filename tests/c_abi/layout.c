/* Prints sizeof and the offset of every field of the ABI structs, one per
 * line ("struct field offset" and "struct sizeof size"), for the binding
 * layout test. */
#include <stddef.h>
#include <stdio.h>

#include "zero_adam.h"

int main(void) {
    printf("zero_adam_hparams sizeof %zu\n", sizeof(zero_adam_hparams));
    printf("zero_adam_hparams lr %zu\n", offsetof(zero_adam_hparams, lr));
    printf("zero_adam_hparams beta1 %zu\n", offsetof(zero_adam_hparams, beta1));
    printf("zero_adam_hparams beta2 %zu\n", offsetof(zero_adam_hparams, beta2));
    printf("zero_adam_hparams eps %zu\n", offsetof(zero_adam_hparams, eps));
    printf("zero_adam_hparams weight_decay %zu\n", offsetof(zero_adam_hparams, weight_decay));
    printf("zero_ctrl sizeof %zu\n", sizeof(zero_ctrl));
    printf("zero_ctrl step %zu\n", offsetof(zero_ctrl, step));
    printf("zero_ctrl skipped %zu\n", offsetof(zero_ctrl, skipped));
    printf("zero_ctrl loss_scale %zu\n", offsetof(zero_ctrl, loss_scale));
    printf("zero_ctrl growth_tracker %zu\n", offsetof(zero_ctrl, growth_tracker));
    printf("zero_ctrl parity %zu\n", offsetof(zero_ctrl, parity));
    printf("zero_ctrl last_skipped %zu\n", offsetof(zero_ctrl, last_skipped));
    printf("zero_ctrl device_error %zu\n", offsetof(zero_ctrl, device_error));
    printf("zero_ctrl reserved %zu\n", offsetof(zero_ctrl, reserved));
    printf("zero_step_args sizeof %zu\n", sizeof(zero_step_args));
    printf("zero_step_args P %zu\n", offsetof(zero_step_args, P));
    printf("zero_step_args R %zu\n", offsetof(zero_step_args, R));
    printf("zero_step_args owner %zu\n", offsetof(zero_step_args, owner));
    printf("zero_step_args grad_dtype %zu\n", offsetof(zero_step_args, grad_dtype));
    printf("zero_step_args param_dtype %zu\n", offsetof(zero_step_args, param_dtype));
    printf("zero_step_args grads %zu\n", offsetof(zero_step_args, grads));
    printf("zero_step_args rank_weights %zu\n", offsetof(zero_step_args, rank_weights));
    printf("zero_step_args master %zu\n", offsetof(zero_step_args, master));
    printf("zero_step_args exp_avg %zu\n", offsetof(zero_step_args, exp_avg));
    printf("zero_step_args exp_avg_sq %zu\n", offsetof(zero_step_args, exp_avg_sq));
    printf("zero_step_args params16 %zu\n", offsetof(zero_step_args, params16));
    printf("zero_step_args reduced_out %zu\n", offsetof(zero_step_args, reduced_out));
    printf("zero_step_args hp %zu\n", offsetof(zero_step_args, hp));
    printf("zero_step_args check_nonfinite %zu\n", offsetof(zero_step_args, check_nonfinite));
    printf("zero_step_args growth_interval %zu\n", offsetof(zero_step_args, growth_interval));
    printf("zero_step_args ctrl %zu\n", offsetof(zero_step_args, ctrl));
    printf("zero_step_args workspace %zu\n", offsetof(zero_step_args, workspace));
    printf("zero_step_args state_offset %zu\n", offsetof(zero_step_args, state_offset));
    printf("zero_step_args n_push %zu\n", offsetof(zero_step_args, n_push));
    printf("zero_step_args path %zu\n", offsetof(zero_step_args, path));
    printf("zero_step_args push_params16 %zu\n", offsetof(zero_step_args, push_params16));
    printf("zero_step_args n_grads %zu\n", offsetof(zero_step_args, n_grads));
    printf("zero_step_args reserved2 %zu\n", offsetof(zero_step_args, reserved2));
    printf("zero_step_args grad_offset %zu\n", offsetof(zero_step_args, grad_offset));
    printf("zero_accum_args sizeof %zu\n", sizeof(zero_accum_args));
    printf("zero_accum_args P %zu\n", offsetof(zero_accum_args, P));
    printf("zero_accum_args R %zu\n", offsetof(zero_accum_args, R));
    printf("zero_accum_args owner %zu\n", offsetof(zero_accum_args, owner));
    printf("zero_accum_args grad_dtype %zu\n", offsetof(zero_accum_args, grad_dtype));
    printf("zero_accum_args first %zu\n", offsetof(zero_accum_args, first));
    printf("zero_accum_args grads %zu\n", offsetof(zero_accum_args, grads));
    printf("zero_accum_args rank_weights %zu\n", offsetof(zero_accum_args, rank_weights));
    printf("zero_accum_args accum %zu\n", offsetof(zero_accum_args, accum));
    printf("zero_accum_args scale %zu\n", offsetof(zero_accum_args, scale));
    printf("zero_accum_args workspace %zu\n", offsetof(zero_accum_args, workspace));
    printf("zero_accum_args ctrl %zu\n", offsetof(zero_accum_args, ctrl));
    printf("zero_accum_args path %zu\n", offsetof(zero_accum_args, path));
    printf("zero_accum_args accum_offset %zu\n", offsetof(zero_accum_args, accum_offset));
    printf("zero_tensor_list sizeof %zu\n", sizeof(zero_tensor_list));
    printf("zero_tensor_list table %zu\n", offsetof(zero_tensor_list, table));
    printf("zero_tensor_list P %zu\n", offsetof(zero_tensor_list, P));
    printf("zero_tensor_list T %zu\n", offsetof(zero_tensor_list, T));
    printf("zero_tensor_list R %zu\n", offsetof(zero_tensor_list, R));
    printf("zero_tensor_list grad_dtype %zu\n", offsetof(zero_tensor_list, grad_dtype));
    printf("zero_tensor_list param_dtype %zu\n", offsetof(zero_tensor_list, param_dtype));
    printf("zero_tensor_list table_bytes %zu\n", offsetof(zero_tensor_list, table_bytes));
    return 0;
}
