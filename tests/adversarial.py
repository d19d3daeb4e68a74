"""Adversarial inputs for the prefill's +-s operand with bf16 x (input generation only; no
expected value is computed here).

bf16 keeps 8 significant bits, an fp16 scale has 11. An fp16 scale whose last three mantissa
bits are 100 sits exactly halfway between two bf16 values, so rounding it to bf16 moves it by
2^-8 of its value, twice the 2e-3 relative tolerance on sum |x s|. With a group whose weights
all have the same sign and x all positive, every term then errs the same way."""

import torch

import synth

# fp16 bit patterns on bf16 rounding ties in many binades, from the subnormal 0x0202 (its
# 10 significant bits end in 10) to 0x5014 = 32.625 (normal ones: low three mantissa bits
# 100); 0x3C04 = 1.00390625.
TIE_SCALES = [0x3C04, 0x2C04, 0x1C04, 0x4C04, 0x340C, 0x0C04, 0x0202, 0x5014, 0x2424, 0x3844]


def _scales(N, K):
    G = K // 128
    idx = torch.arange(N * G, dtype=torch.int64).reshape(N, G)
    bits = torch.tensor(TIE_SCALES, dtype=torch.int64)[(idx * 7 + idx // G) % len(TIE_SCALES)]
    return bits.to(torch.int16).view(torch.float16)


def _group_kind(N, K):
    """Per (row, group): 0 all-ones / all +1, 1 all-zeros / all -1, 2 random."""
    G = K // 128
    idx = torch.arange(N * G, dtype=torch.int64).reshape(N, G)
    return (idx * 5 + idx // G) % 3


def adversarial_binary(N, K):
    """(words int32 [N, K/32], scales fp16 [N, K/128])."""
    kind = _group_kind(N, K).repeat_interleave(4, dim=1)            # 4 words per group
    rnd = synth.binary_words(77, N, K)
    words = torch.where(kind == 0, torch.full_like(rnd, -1), torch.where(kind == 1, torch.zeros_like(rnd), rnd))
    return words.contiguous(), _scales(N, K)


def adversarial_ternary_q(N, K):
    """(q int8 [N, K] in {-1, 0, +1}, scales fp16 [N, K/128])."""
    kind = _group_kind(N, K).repeat_interleave(128, dim=1)
    rnd = synth.random_ternary(78, synth.TID_TERNARY, (N, K))
    q = torch.where(kind == 0, torch.ones_like(rnd), torch.where(kind == 1, -torch.ones_like(rnd), rnd))
    return q.contiguous(), _scales(N, K)


def positive_bf16_x(seed, M, K):
    """Strictly positive bf16 activations: |N(0, 1)| + 0.05."""
    return (synth.activations(seed, M, K, dtype=torch.float32).abs() + 0.05).to(torch.bfloat16)


def wide_range_bf16_x(seed, M, K):
    """bf16 rows of |N(0, 1)| + 0.05 scaled by 2^(-100 + 2 m mod 201); every 16th row is zero."""
    x = synth.activations(seed, M, K, dtype=torch.float32).abs().double() + 0.05
    e = (-100 + (2 * torch.arange(M, dtype=torch.int64)) % 201).double()
    x = x * torch.pow(2.0, e)[:, None]
    x[::16] = 0.0
    return x.to(torch.bfloat16)
