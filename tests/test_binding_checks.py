"""The binding's extent and dtype checks (host only: no device, no library
call).  The C ABI receives raw pointers and cannot see extents, so a tensor of
the wrong shape or dtype must be refused before the call."""

import pytest
import torch

import moe_grouped_gemm_act_b200 as dg


def ops(m=200, n=264, k=512, ld=None):
    ld = ld or -(-m // 4) * 4
    return (torch.zeros((m, k), dtype=torch.uint8), torch.zeros((k // 128, ld)),
            torch.zeros((n, k), dtype=torch.uint8), torch.zeros((-(-n // 128), k // 128)))


def test_good_operands_pass():
    dg._gemm_operands(*ops(), 200, 264, 512)
    dg._expect(torch.zeros((200, 264), dtype=torch.bfloat16), "d", torch.bfloat16, (200, 264))


@pytest.mark.parametrize("which,bad", [
    (0, torch.zeros((200, 384), dtype=torch.uint8)),      # A with the wrong K
    (0, torch.zeros((200, 512), dtype=torch.int8)),       # A of the wrong dtype
    (1, torch.zeros((4, 198))),                           # ld of alpha not a multiple of 4
    (1, torch.zeros((4, 196))),                           # ld of alpha < M
    (1, torch.zeros((3, 200))),                           # too few K groups
    (2, torch.zeros((256, 512), dtype=torch.uint8)),      # B with the wrong N
    (3, torch.zeros((2, 4))),                             # beta short by one N block
    (3, torch.zeros((3, 4), dtype=torch.float64)),        # beta of the wrong dtype
])
def test_bad_operand_refused(which, bad):
    args = list(ops())
    args[which] = bad
    with pytest.raises(ValueError):
        dg._gemm_operands(*args, 200, 264, 512)


def test_grouped_and_batched_operands():
    g, m, n, k = 3, 130, 136, 256
    a = torch.zeros((g, m, k), dtype=torch.uint8)
    sfa = torch.zeros((g, k // 128, 132))
    b = torch.zeros((g, n, k), dtype=torch.uint8)
    sfb = torch.zeros((g, 2, k // 128))
    dg._gemm_operands(a, sfa, b, sfb, m, n, k, groups=g, a_batch=g)
    with pytest.raises(ValueError):   # one expert's weights missing
        dg._gemm_operands(a, sfa, b[:2], sfb, m, n, k, groups=g, a_batch=g)
    with pytest.raises(ValueError):   # masked scales without the expert axis
        dg._gemm_operands(a, sfa[0], b, sfb, m, n, k, groups=g, a_batch=g)


def test_output_checks():
    with pytest.raises(ValueError):
        dg._expect(torch.zeros((200, 256), dtype=torch.bfloat16), "d", torch.bfloat16, (200, 264))
    with pytest.raises(ValueError):
        dg._expect(torch.zeros((200, 264)), "d", torch.bfloat16, (200, 264))
    with pytest.raises(ValueError):
        dg._expect(None, "c", torch.float32, (200, 264))


def test_k_off_the_grid_is_left_to_the_c_abi():
    # K % 128 != 0 is reported by the library itself (DG_ERR_INVALID_ARG)
    a, sfa, b, sfb = ops(k=512)
    dg._gemm_operands(a[:, :200], sfa, b[:, :200], sfb, 200, 264, 200)
