"""Bytes and bits per parameter of the NF4 + double-quant storage format.
Test infrastructure: see ``oracle/__init__``.

The pages work the format's memory bill by hand [P1 "Summary"; P2 "Break the
name into two parts"; P3 "Worked example"; P4 "The three ideas behind QLoRA",
2. Double quantization; P5 figures 4 and 5].  These functions state the sizes
of the three buffers the format stores for ``numel`` weights (a multiple of
64): packed codes, one uint8 absmax code per block of 64, one fp32 constant
per group of 256 blocks.
"""

BLOCK = 64
GROUP = 256


def n_blocks(numel: int) -> int:
    if numel % BLOCK:
        raise ValueError("numel must be a multiple of 64")
    return numel // BLOCK


def n_groups(numel: int) -> int:
    return (n_blocks(numel) + GROUP - 1) // GROUP


def code_bytes(numel: int) -> int:
    """Packed 4-bit codes: two per byte."""
    return numel // 2


def absmax_fp32_bytes(numel: int) -> int:
    """Single quantization: one fp32 absmax per block of 64."""
    return 4 * n_blocks(numel)


def absmax_dq_bytes(numel: int) -> int:
    """Double quantization: one uint8 per block plus one fp32 per 256 blocks."""
    return n_blocks(numel) + 4 * n_groups(numel)


def total_bytes(numel: int, double_quant: bool = True) -> int:
    scales = absmax_dq_bytes(numel) if double_quant else absmax_fp32_bytes(numel)
    return code_bytes(numel) + scales


def bits_per_param(numel: int, double_quant: bool = True) -> float:
    return 8.0 * total_bytes(numel, double_quant) / numel


def scale_bits_per_param(numel: int, double_quant: bool = True) -> float:
    b = absmax_dq_bytes(numel) if double_quant else absmax_fp32_bytes(numel)
    return 8.0 * b / numel


# Per-parameter rates of the format in the limit of many groups.
RATE_CODES = 4.0                                        # bits
RATE_SCALE_FP32 = 32.0 / BLOCK                          # 0.5 bit
RATE_SCALE_DQ = 8.0 / BLOCK + 32.0 / (BLOCK * GROUP)    # 0.126953125 bit
