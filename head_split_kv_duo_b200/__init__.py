"""B200-native hybrid-head KV attention (DuoAttention's retrieval / streaming heads).

``head_split_kv_duo_b200.duo`` is the Python binding of the C-ABI library
``libduo.so`` (``include/duo.h``); ``head_split_kv_duo_b200.inputs`` holds the
seeded synthetic input generators.  Importing the package loads nothing.
"""
__all__ = ["duo", "inputs"]
__version__ = "0.1.0"
