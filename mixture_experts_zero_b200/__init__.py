"""B200-native forward pass of a MoE layer with zero-computation experts, and its expert-bias
update (LongCat-Flash llm-wiki entity page, section 2.1).

The compute path is the C-ABI library ``libmoezero.so`` (hand-written sm_100a CUDA kernels);
this package only marshals torch tensors to it. The library is loaded on first use, and a
missing library raises instead of falling back to anything else.
"""
